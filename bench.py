#!/usr/bin/env python
"""Benchmark of the paged KV-cache hot path on B200.

One step = one pass of the hot path over one batch of the 4k-token decode
workload (batch 16 x 4096 tokens, 32 q / 8 KV heads, head_dim 128, block 16,
bf16): copy-on-write block copy (none are due in this workload: no block is
shared), the KV-cache append of the batch's 16 new tokens, then paged decode
attention over all 4096 tokens of every request (the append inside the decode
launch).  Inputs are synthetic (seeded N(0,1) values, randomly permuted block
pool) and resident in HBM before the timed region.  Each step uses the next
of 4 layer pools (268 MB of K+V each, 1.07 GB in all), so every step reads KV
that is not in the 126 MB L2; the 32 steps of a 32-layer model's decode
iteration form one CUDA graph.

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle (the
only other implementation of the path) on a bounded sample instead.

Usage: python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
Multi-GPU: launched by torchrun, one rank per GPU; every rank runs its own
replica (independent requests, no data-path collective), timing is the max
over ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode attention KV GB/s (fraction of HBM peak) and tokens/s at 1 B200"
UNIT = "GB/s"
WORKLOAD = "gqa_4k: batch 16 x 4096 tokens, 32 q / 8 KV heads, head_dim 128, block 16, bf16"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0  # the B200's ~8 TB/s HBM3e figure, for the nominal fraction
ROOFLINE_LAUNCHES = 2000  # decode-append launches timed for the roofline, whatever --steps
DEC_RUN = 20               # back-to-back decode-append launches per timed graph (roofline)
ISOLATED_LAUNCHES = 200    # single decode-append launches timed on their own (latency)
SEPARATE_SWEEPS = 10       # iterations timed for the step with the append as its own launch
N_LAYERS = 4               # distinct K/V pools (1.07 GB together: every step reads HBM)
STEPS_PER_GRAPH = 32       # steps of one decode iteration of a 32-layer model, one CUDA graph
DECODE_SRC = os.path.join(ROOT, "paged_kv_cache_412_b200", "csrc", "decode_mma.cu")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "decode_gqa_4k_traffic.txt")


# ---------------------------------------------------------------------------
# byte model of one step (the decode's algorithmic bytes; the append's bytes
# are reported beside it)
# ---------------------------------------------------------------------------

def decode_bytes(B, L, Hq, Hkv, d, e_kv=2, e_q=2, e_out=2):
    """K and V of every token once per kv head, plus q and out."""
    return 2 * B * L * Hkv * d * e_kv + B * Hq * d * (e_q + e_out)


def write_bytes(T, Hkv, d, e=2):
    """Read the new K and V rows, write them into the cache."""
    return 2 * 2 * T * Hkv * d * e


def measured_peak():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def traffic_per_launch():
    """DRAM bytes per decode launch from the committed ncu summary, or None if
    the summary is missing or was taken on a different kernel source."""
    try:
        src_hash = hashlib.sha256(open(DECODE_SRC, "rb").read()).hexdigest()[:16]
        vals = {}
        for line in open(TRAFFIC_FILE):
            if "=" in line and not line.lstrip().startswith("#"):
                k, v = line.split("=", 1)
                vals[k.strip()] = v.split("#")[0].strip()
        if vals.get("decode_source_sha256_16") != src_hash:
            return None
        return int(float(vals["dram_bytes_per_launch"]))
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clock/throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, path: str | None = None):
        import tempfile
        self.gpu = gpu_index
        self.proc = None
        self.path = path or os.path.join(tempfile.gettempdir(), f"pkv_clocks_gpu{gpu_index}.csv")

    def start(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------------------
# distributed plumbing (only for --gpus > 1 under torchrun)
# ---------------------------------------------------------------------------

def replica_seed(rank: int, layer: int) -> int:
    """Seed of a rank's replica of one layer pool: every rank decodes its own
    independent batch (weak scaling, no data exchanged between ranks)."""
    return 1002 + 100 * rank + layer


def relaunch_under_torchrun(n_gpus: int, argv: list[str]) -> int:
    """``--gpus N`` (N > 1) run without torchrun: start N ranks of this script
    under torch.distributed.run on 127.0.0.1 and return their exit status."""
    import socket
    with socket.socket() as sk:
        sk.bind(("127.0.0.1", 0))
        port = sk.getsockname()[1]
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1",
           f"--nproc-per-node={n_gpus}", "--master-addr=127.0.0.1", f"--master-port={port}",
           os.path.abspath(__file__), *argv]
    return subprocess.call(cmd)


def dist_setup(n_gpus: int):
    """Rank, world size and local rank of this process.  The world must be the
    requested --gpus: a mismatch is an error, never a silent single replica."""
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != n_gpus:
        raise SystemExit(f"bench.py: --gpus {n_gpus} but WORLD_SIZE is {world}; launch one "
                         f"process per GPU (torchrun --nproc-per-node {n_gpus}), or run "
                         f"without torchrun and let bench.py start the ranks")
    if world > 1:
        import datetime
        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if torch.cuda.is_available():
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(0)
    return rank, world, local


def dist_max(value: float, world: int) -> float:
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    t = torch.tensor([value], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def dist_done(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


# ---------------------------------------------------------------------------
# CPU baseline: the oracle, as it stands, on a bounded sample
# ---------------------------------------------------------------------------

_ALL_CORES = None


def oracle_all_cores(lib) -> int:
    """The oracle's thread count with nothing set (all host cores, or
    OMP_NUM_THREADS), read once: a single-thread timing sets the OpenMP
    default of this thread to 1, so every call passes its count explicitly."""
    global _ALL_CORES
    if _ALL_CORES is None:
        import oracle
        _ALL_CORES = oracle.max_threads(lib)
    return _ALL_CORES


def cpu_baseline(budget_s: float = 12.0, per_call_cap_s: float | None = None) -> dict:
    """Time the oracle (write + decode) on whole requests of the same workload
    until about ``budget_s`` seconds of CPU work; report KV GB/s by the same
    byte formula as the GPU line."""
    import oracle
    import workloads
    w = workloads.gqa_4k(poison=False, seed=2002, batch=4)
    lib = oracle.load()
    threads = oracle_all_cores(lib)
    total_bytes = 0
    calls = 0
    reqs = 0
    t_all = 0.0
    while t_all < budget_s:
        b = calls % w.B
        sl = slice(b, b + 1)
        kc, vc = w.k_cache, w.v_cache
        t0 = time.perf_counter()
        oracle.kv_cache_write(w.k_new[sl], w.v_new[sl], w.slot_mapping[sl], kc, vc, lib=lib)
        oracle.decode(w.q[sl], kc, vc, w.block_tables[sl], w.seq_lens[sl], w.scale,
                      nthreads=threads, lib=lib)
        t_all += time.perf_counter() - t0
        total_bytes += decode_bytes(1, 4096, 32, 8, 128)
        calls += 1
        reqs += 1
        if per_call_cap_s is not None and t_all > per_call_cap_s:
            break
    gbs = total_bytes / t_all / 1e9
    one = _oracle_rate(w, 1, 3.0, lib, per_head=True)
    return {"value": round(gbs, 4), "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{reqs} whole requests of the 4k workload (4096 tokens x 32 q / 8 KV "
                      f"heads each), fp64 C oracle with OpenMP over (request, head), "
                      f"{t_all:.1f} s of CPU time",
            "seconds": round(t_all, 3),
            "single_thread": {"value": one["GBps"], "unit": UNIT, "cores": 1,
                              "sample": f"{one['sample']} of the 4k workload (one kv head's "
                                        f"4 query heads x 4096 tokens each)"}}


def run_reference(args, rank: int, world: int):
    """--impl reference: the CPU oracle on a bounded sample per step."""
    if rank != 0:
        return
    import oracle
    import workloads
    w = workloads.gqa_4k(poison=False, seed=2002, batch=4)
    lib = oracle.load()
    threads = oracle_all_cores(lib)
    budget_total = 150.0
    per_step = max(budget_total / max(args.steps + args.warmup, 1), 0.0)
    # calibrate the sample: whole requests if affordable, else the first
    # kv-head group(s) of one request (all 4096 tokens)
    b = 0
    sl = slice(0, 1)
    t0 = time.perf_counter()
    oracle.decode(w.q[sl], w.k_cache, w.v_cache, w.block_tables[sl], w.seq_lens[sl], w.scale,
                  lib=lib)
    t_req = time.perf_counter() - t0
    G = w.Hq // w.Hkv
    if per_step >= t_req:
        nreq = max(1, min(w.B, int(per_step // t_req)))
        groups = w.Hkv
    else:
        nreq = 1
        groups = max(1, min(w.Hkv, int(per_step / (t_req / w.Hkv))))
    # sub-problem for `groups` kv heads: slice the cache's kv-head axis once
    kc = np.ascontiguousarray(w.k_cache[:, :groups])
    vc = np.ascontiguousarray(w.v_cache[:, :groups])
    q = np.ascontiguousarray(w.q[:nreq, : groups * G])
    knew = np.ascontiguousarray(w.k_new[:nreq, :groups])
    vnew = np.ascontiguousarray(w.v_new[:nreq, :groups])
    bt, sls, sm = w.block_tables[:nreq], w.seq_lens[:nreq], w.slot_mapping[:nreq]

    def step():
        oracle.kv_cache_write(knew, vnew, sm, kc, vc, lib=lib)
        oracle.decode(q, kc, vc, bt, sls, w.scale, lib=lib)

    for _ in range(args.warmup):
        step()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        step()
    dt = time.perf_counter() - t0
    step_bytes = decode_bytes(nreq, 4096, groups * G, groups, 128)
    value = step_bytes * args.steps / dt / 1e9
    sample = (f"{nreq} request(s) x {groups} of 8 kv-head groups ({groups * G} q heads) x "
              f"4096 tokens per step")
    line = {"impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(dt / args.steps * 1e3, 4), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": WORKLOAD, "sample": sample, "l2": "n/a (host)"},
            "cpu_baseline": {"value": round(value, 4), "unit": UNIT, "cores": threads,
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 4), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "tokens_per_s": round(nreq * args.steps / dt, 3)}
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------

def run_ours(args, rank: int, world: int, local: int):
    import torch
    import paged_kv_cache_412_b200 as pkv
    import workloads

    dev = torch.device("cuda", local if world > 1 else 0)
    torch.cuda.set_device(dev)
    B, L, Hq, Hkv, d, bs = 16, 4096, 32, 8, 128, 16

    # --- inputs resident in HBM: N_LAYERS layer pools of the same workload ---
    layers = []
    for li in range(N_LAYERS):
        w = workloads.gqa_4k(poison=False, seed=replica_seed(rank, li))
        t = {}
        t["q"] = torch.from_numpy(w.q.view(np.int16)).to(dev).view(torch.bfloat16)
        t["kc"] = torch.from_numpy(w.k_cache.view(np.int16)).to(dev).view(torch.bfloat16)
        t["vc"] = torch.from_numpy(w.v_cache.view(np.int16)).to(dev).view(torch.bfloat16)
        t["bt"] = torch.from_numpy(w.block_tables).to(dev)
        t["sl"] = torch.from_numpy(w.seq_lens).to(dev)
        t["kn"] = torch.from_numpy(w.k_new.view(np.int16)).to(dev).view(torch.bfloat16)
        t["vn"] = torch.from_numpy(w.v_new.view(np.int16)).to(dev).view(torch.bfloat16)
        t["sm"] = torch.from_numpy(w.slot_mapping).to(dev)
        t["host"] = w
        layers.append(t)
        del w
    out = torch.empty((B, Hq, d), dtype=torch.bfloat16, device=dev)
    ws_bytes = pkv.decode_workspace_bytes(B, Hq, Hkv, d, bs, L, 0)
    ws = pkv.new_workspace(ws_bytes, dev)
    no_pairs = torch.empty((0, 2), dtype=torch.int64, device=dev)
    scale = 1.0 / math.sqrt(d)

    # Every request appends one token, so the step's new rows are one per
    # request ([B, Hkv, d]) and the append rides in the decode launch
    # (paged_attention_decode_append); ``fused=False`` is the same step with
    # the append as its own kv_cache_write launch.
    def step_body(t, with_write=True, fused=True):
        if with_write:
            pkv.copy_blocks(t["kc"], t["vc"], no_pairs)  # no shared block to fork here
            if fused:
                pkv.paged_attention_decode_append(t["q"], t["kn"], t["vn"], t["kc"], t["vc"],
                                                  t["bt"], t["sl"], bs, scale, out,
                                                  max_seq_len=L, workspace=ws)
                return
            pkv.kv_cache_write(t["kn"], t["vn"], t["sm"], t["kc"], t["vc"])
        pkv.paged_attention_decode(t["q"], t["kc"], t["vc"], t["bt"], t["sl"], bs, scale, out,
                                   max_seq_len=L, workspace=ws)

    # eager warm-up (first calls set up per-device state outside any capture)
    for i in range(args.warmup):
        step_body(layers[i % N_LAYERS])
    step_body(layers[0], fused=False)
    torch.cuda.synchronize()
    assert pkv.get_device_error() == 0

    # A decode iteration of a model runs the step once per layer, back to
    # back: one CUDA graph holds the STEPS_PER_GRAPH steps of an iteration of
    # a 32-layer model (layer l reads pool l % N_LAYERS, which the three other
    # pools have evicted from L2 since its last visit), so consecutive kernels
    # overlap through programmatic dependent launch as they would in the
    # serving loop; a second graph holds the first K % STEPS_PER_GRAPH steps.
    def capture(steps, with_write, fused=True):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            for li in range(steps):
                step_body(layers[li % N_LAYERS], with_write, fused)
        return g
    sweep = capture(STEPS_PER_GRAPH, True)
    n_sweeps, rest = divmod(args.steps, STEPS_PER_GRAPH)
    part = capture(rest, True) if rest else None
    for _ in range(max(1, -(-args.warmup // STEPS_PER_GRAPH))):
        sweep.replay()
    if part is not None:  # a graph's first launch also uploads it: not inside the timing
        part.replay()
    torch.cuda.synchronize()

    # --- timed region: K steps (graph replays), device-timed ---
    sampler = ClockSampler(dev.index if dev.index is not None else 0, args.clocks_csv or None)
    bounds = [torch.cuda.Event(enable_timing=True) for _ in range(n_sweeps + 2)]
    sampler.start()
    time.sleep(0.3)
    # the sampler's start-up left the GPU idle: one more warm-up replay, so the
    # timed region starts on a busy GPU
    (part if part is not None and n_sweeps == 0 else sweep).replay()
    dist_barrier(world)
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_push("timed steps")
    bounds[0].record()
    for i in range(n_sweeps):
        sweep.replay()
        bounds[i + 1].record()
    if part is not None:
        part.replay()
    bounds[n_sweeps + 1].record()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    dist_barrier(world)
    clocks = sampler.stop()
    ms_total = bounds[0].elapsed_time(bounds[-1])
    # per-step time of each full sweep (the partial sweep only counts in the total)
    step_ms = [bounds[i].elapsed_time(bounds[i + 1]) / STEPS_PER_GRAPH for i in range(n_sweeps)] or \
              [ms_total / args.steps]
    ms_total_max = dist_max(ms_total, world)
    ms_step = ms_total_max / args.steps
    del sweep, part

    # The same step with the append as its own launch (kv_cache_write, then
    # the decode): graphs of STEPS_PER_GRAPH steps, events around each.
    sep = capture(STEPS_PER_GRAPH, True, fused=False)
    for _ in range(3):
        sep.replay()
    torch.cuda.synchronize()
    sep_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(SEPARATE_SWEEPS)]
    for a, b in sep_ev:
        a.record()
        sep.replay()
        b.record()
    torch.cuda.synchronize()
    sep_ms = statistics.median(a.elapsed_time(b) / STEPS_PER_GRAPH for a, b in sep_ev)
    del sep
    assert pkv.get_device_error() == 0

    # --- the decode kernel alone (roofline), a fixed number of launches ---
    # Throughput: graphs of DEC_RUN back-to-back decode launches over the layer
    # pools, events around each graph; the launch duration is the graph's time
    # over DEC_RUN.  Latency of one launch on its own (events around a graph
    # of one launch) is reported beside it.
    dec_run = capture(DEC_RUN, True)
    dec_one = [capture(1, True) for _ in range(1)]
    n_runs = -(-ROOFLINE_LAUNCHES // DEC_RUN)
    n_dec = n_runs * DEC_RUN
    for _ in range(3):
        dec_run.replay()
    torch.cuda.synchronize()
    dev_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n_runs)]
    torch.cuda.nvtx.range_push("roofline: back-to-back decode-append launches")
    for a, b in dev_ev:
        a.record()
        dec_run.replay()
        b.record()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    decode_ms = [a.elapsed_time(b) / DEC_RUN for a, b in dev_ev]
    iso_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(ISOLATED_LAUNCHES)]
    torch.cuda.nvtx.range_push("decode launches on their own")
    for a, b in iso_ev:
        a.record()
        dec_one[0].replay()
        b.record()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    iso_ms = statistics.fmean(a.elapsed_time(b) for a, b in iso_ev)
    del dec_run, dec_one
    # the decode alone (no append), for comparison
    dec_only = capture(DEC_RUN, False)
    for _ in range(3):
        dec_only.replay()
    torch.cuda.synchronize()
    for a, b in dev_ev:
        a.record()
        dec_only.replay()
        b.record()
    torch.cuda.synchronize()
    dec_only_ms = statistics.fmean(a.elapsed_time(b) / DEC_RUN for a, b in dev_ev)
    del dec_only

    dbytes = decode_bytes(B, L, Hq, Hkv, d)
    wbytes = write_bytes(B, Hkv, d)
    value = dbytes * args.steps * world / (ms_total_max / 1e3) / 1e9
    dec_avg_ms = statistics.fmean(decode_ms)
    dec_med_ms = statistics.median(decode_ms)
    peak, peak_kind = measured_peak()
    # the fused launch moves the decode's bytes and the append's (k_new and
    # v_new read, the same bytes written to the cache)
    achieved = (dbytes + wbytes) / (dec_avg_ms / 1e3) / 1e9

    # --- e2e: host inputs -> device, the step, result -> host, per step ---
    t0l = layers[0]
    hw = t0l["host"]
    # A step's inputs staged in one pinned buffer and moved with one copy (one
    # copy's fixed cost instead of six); the device side is typed views of one
    # buffer, each part 256-byte aligned.
    parts = [("q", hw.q.view(np.int16), torch.bfloat16),
             ("kn", hw.k_new.view(np.int16), torch.bfloat16),
             ("vn", hw.v_new.view(np.int16), torch.bfloat16),
             ("bt", hw.block_tables, torch.int32), ("sl", hw.seq_lens, torch.int32)]
    offs, total = {}, 0
    for name, arr, _ in parts:
        offs[name] = total
        total += (arr.nbytes + 255) // 256 * 256
    h_in = torch.zeros(total, dtype=torch.uint8).pin_memory()
    d_in = torch.empty(total, dtype=torch.uint8, device=dev)
    views = {}
    for name, arr, tdt in parts:
        o, n = offs[name], arr.nbytes
        h_in[o:o + n].copy_(torch.from_numpy(np.ascontiguousarray(arr).view(np.uint8).ravel()))
        views[name] = d_in[o:o + n].view(tdt).view(arr.shape)
    h_out = torch.empty((B, Hq, d), dtype=torch.int16).pin_memory()
    h2d = total
    d2h = h_out.numel() * h_out.element_size()

    def e2e_body(li):
        t = layers[li % N_LAYERS]
        d_in.copy_(h_in, non_blocking=True)
        pkv.copy_blocks(t["kc"], t["vc"], no_pairs)
        pkv.paged_attention_decode_append(views["q"], views["kn"], views["vn"], t["kc"],
                                          t["vc"], views["bt"], views["sl"], bs, scale, out,
                                          max_seq_len=L, workspace=ws)
        h_out.copy_(out.view(torch.int16), non_blocking=True)

    # A serving loop captures its decode step once and replays it: one graph per
    # layer pool holding the host->device copies, the three calls and the
    # device->host copy; every step is a replay plus a stream synchronize.
    e2e_mode = ("CUDA graph per step (one copy in of the staged inputs, copy_blocks, "
                "decode with the fused append, copy out)")
    try:
        e2e_graphs = []
        for li in range(N_LAYERS):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                e2e_body(li)
            e2e_graphs.append(g)

        def e2e_step(li):
            e2e_graphs[li % N_LAYERS].replay()
            torch.cuda.current_stream().synchronize()
    except Exception as ex:  # capture refused: the same calls issued eagerly
        e2e_mode = f"eager calls (graph capture failed: {type(ex).__name__})"

        def e2e_step(li):
            e2e_body(li)
            torch.cuda.current_stream().synchronize()

    e2e_steps = max(10, min(args.steps, 2000))
    for i in range(5):
        e2e_step(i)
    dist_barrier(world)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.nvtx.range_push("e2e: graph per step")
    e0.record()
    for i in range(e2e_steps):
        e2e_step(i)
    e1.record()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    e2e_ms = dist_max(e0.elapsed_time(e1), world)
    e2e_value = dbytes * e2e_steps * world / (e2e_ms / 1e3) / 1e9
    assert pkv.get_device_error() == 0

    # The same step with the two C-ABI calls issued eagerly every step: each
    # call's host validation, planning, tensor-map encoding and launch is inside
    # the timed region.  host_us_per_step is the host time of those calls.
    def eager_step(li):
        e2e_body(li)
        torch.cuda.current_stream().synchronize()
    for i in range(5):
        eager_step(i)
    dist_barrier(world)
    torch.cuda.synchronize()
    host_s = 0.0
    torch.cuda.nvtx.range_push("e2e: eager calls")
    e0.record()
    for i in range(e2e_steps):
        h0 = time.perf_counter()
        e2e_body(i)
        host_s += time.perf_counter() - h0
        torch.cuda.current_stream().synchronize()
    e1.record()
    torch.cuda.synchronize()
    torch.cuda.nvtx.range_pop()
    eager_ms = dist_max(e0.elapsed_time(e1), world)
    eager_value = dbytes * e2e_steps * world / (eager_ms / 1e3) / 1e9
    assert pkv.get_device_error() == 0
    del e2e_graphs

    configs = None
    if world == 1 and not args.no_configs:
        layers.clear()  # free the four layer pools before the per-workload section
        torch.cuda.empty_cache()
        configs = run_configs(pkv, torch, dev, peak, peak_kind,
                              with_oracle=not args.no_cpu_baseline)

    result = None
    if rank == 0:
        cpu = cpu_baseline() if (world == 1 and not args.no_cpu_baseline) else None
        result = {
            "metric": METRIC, "value": round(value, 2), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": WORKLOAD, "global_batch": B * world, "seq_len": L,
                       "num_q_heads": Hq, "num_kv_heads": Hkv, "head_dim": d, "block_size": bs,
                       "layers_rotated": N_LAYERS, "steps_per_graph": STEPS_PER_GRAPH,
                       "l2": f"inputs larger than L2: {N_LAYERS} layer pools of "
                             f"{2 * B * L * Hkv * d * 2 / 1e6:.0f} MB K+V rotated per step",
                       "parallelism": f"replica x{world}" if world > 1 else "single GPU",
                       "step": "copy_blocks (0 pairs) + paged_attention_decode_append "
                               "(the 16 new tokens appended inside the decode launch); the "
                               f"{STEPS_PER_GRAPH} steps of a 32-layer model's decode "
                               "iteration (layer l on pool l mod "
                               f"{N_LAYERS}) captured in one CUDA graph, replayed back to back"},
            "tokens_per_s": round(B * world * args.steps / (ms_total_max / 1e3), 1),
            "context_tokens_per_s": round(B * L * world * args.steps / (ms_total_max / 1e3), 1),
            "fraction_of_hbm_peak": round(value / peak, 4),
            "fraction_of_nominal_peak": round(value / NOMINAL_HBM_GBS, 4),
            "nominal_peak_gbs": NOMINAL_HBM_GBS,
            "step_ms_median": round(statistics.median(step_ms), 5),
            "step_separate_calls": {
                "ms_median": round(sep_ms, 5),
                "GBps": round(dbytes / (sep_ms / 1e3) / 1e9, 2),
                "note": "the same step with the append as its own launch (copy_blocks + "
                        "kv_cache_write + paged_attention_decode), median over "
                        f"{SEPARATE_SWEEPS} graphs of {STEPS_PER_GRAPH} steps"},
            "decode_ms_avg": round(dec_avg_ms, 5), "decode_ms_median": round(dec_med_ms, 5),
            "decode_launches_timed": n_dec,
            "decode_only_ms_avg": round(dec_only_ms, 5),
            "decode_isolated": {"ms_avg": round(iso_ms, 5), "launches": ISOLATED_LAUNCHES,
                                "GBps": round(dbytes / (iso_ms / 1e3) / 1e9, 2),
                                "note": "one decode-append launch on its own between events (its "
                                        "launch latency, planning and ramp not overlapped "
                                        "with a previous kernel)"},
            "bytes_per_step": {"decode_algorithmic": dbytes, "append": wbytes},
            "roofline": {"bound": "hbm", "achieved": round(achieved, 2), "peak": peak,
                         "unit": "GB/s", "frac": round(achieved / peak, 4),
                         "traffic": traffic_per_launch(),
                         "kernel": "decode_mma_kernel (split decode with in-kernel merge "
                                   "and the fused append)",
                         "bytes": "decode_algorithmic + append",
                         "duration": f"per-launch mean of graphs of {DEC_RUN} back-to-back "
                                     "decode-append launches over the layer pools (events "
                                     "around each graph), after the timed steps",
                         "peak_kind": f"{peak_kind} HBM copy bandwidth"},
            "cpu_baseline": cpu,
            "e2e": {"value": round(e2e_value, 2), "unit": UNIT, "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "steps": e2e_steps,
                    "ms_per_step": round(e2e_ms / e2e_steps, 5),
                    "note": "pinned host inputs copied in and output copied out every step, "
                            "with a stream synchronize per step",
                    "mode": e2e_mode},
            "e2e_eager": {"value": round(eager_value, 2), "unit": UNIT,
                          "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                          "steps": e2e_steps, "ms_per_step": round(eager_ms / e2e_steps, 5),
                          "host_us_per_step": round(host_s / e2e_steps * 1e6, 2),
                          "note": "the same step with copy_blocks and the decode-append "
                                  "called eagerly through the binding every step "
                                  "(host validation, planning, tensor-map encoding and "
                                  "launches inside the timed region); host_us_per_step = "
                                  "host time of the copy-in, two calls and copy-out"},
            "gpu_launches": args.steps,
            "clocks": clocks,
            "configs": configs,
            "configs_l2": _L2Flush.DESCRIPTION if configs else None,
        }
        print(json.dumps(result), flush=True)
    dist_barrier(world)
    return result


# ---------------------------------------------------------------------------
# --suite: one JSON line per workload of the scope table (not the headline)
# ---------------------------------------------------------------------------

class _L2Flush:
    """Between timed launches: writes a buffer twice the size of L2, then reads
    a second one of the same size.  The write evicts whatever the timed launch
    touched; the read makes the L2 write those dirty lines back before the
    launch starts, so the launch neither finds its data in L2 nor pays for the
    flush's own write-backs."""

    DESCRIPTION = "flushed (256 MB write, then 256 MB read of another buffer) before every timed launch"

    def __init__(self, dev):
        import torch
        self.buf = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
        self.clean = torch.zeros(64 << 20, dtype=torch.float32, device=dev)
        self.acc = torch.zeros((), dtype=torch.float32, device=dev)

    def __call__(self):
        import torch
        self.buf.zero_()
        torch.sum(self.clean, dim=0, out=self.acc)


def _device_clean():
    """Fail fast (before any timed launch) if the library's device error word
    is set: a call that reported an error is not worth timing."""
    import paged_kv_cache_412_b200 as pkv
    flags = pkv.get_device_error()
    if flags:
        raise RuntimeError(f"device error word 0x{flags:x} before timing")


def _time_graph(fn, iters, flush, warm=5):
    """Mean / median device time (ms) of ``fn`` captured in a CUDA graph, L2
    flushed before each launch, CUDA events around each launch."""
    import torch
    for _ in range(2):
        fn()
    torch.cuda.synchronize()
    _device_clean()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    for _ in range(warm):
        flush()
        g.replay()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(iters)]
    for a, b in ev:
        flush()
        a.record()
        g.replay()
        b.record()
    torch.cuda.synchronize()
    ms = [a.elapsed_time(b) for a, b in ev]
    del g
    return statistics.fmean(ms), statistics.median(ms)


B2B_RUN = 20    # launches per graph, back-to-back timing of the suite
B2B_POOLS = 4   # copies of the caches the launches rotate over


def _time_back_to_back(fn, run, reps):
    """Median per-launch time (ms) of graphs of ``run`` launches fn(0) .. fn(run-1)
    issued back to back, CUDA events around each graph."""
    import torch
    for i in range(2):
        fn(i)
    torch.cuda.synchronize()
    _device_clean()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(run):
            fn(i)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(reps)]
    for a, b in ev:
        a.record()
        g.replay()
        b.record()
    torch.cuda.synchronize()
    del g
    return statistics.median(a.elapsed_time(b) / run for a, b in ev)


def _dev_workload(w, dev):
    import torch

    def t(a):
        a = np.ascontiguousarray(a)
        if a.dtype == np.uint16:
            return torch.from_numpy(a.view(np.int16)).to(dev).view(torch.bfloat16)
        return torch.from_numpy(a).to(dev)
    d = {"q": t(w.q), "kc": t(w.k_cache), "vc": t(w.v_cache), "bt": t(w.block_tables),
         "sl": t(w.seq_lens), "kn": t(w.k_new), "vn": t(w.v_new),
         "sm": t(w.slot_mapping.astype(np.int64)),
         "pairs": t(w.copy_pairs.astype(np.int64).reshape(-1, 2))}
    d["ks"] = None if w.k_scale is None else t(w.k_scale)
    d["vs"] = None if w.v_scale is None else t(w.v_scale)
    return d


def run_suite(args):
    import torch
    import paged_kv_cache_412_b200 as pkv
    import workloads

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    peak, peak_kind = measured_peak()
    flush = _L2Flush(dev)
    iters = max(20, min(args.steps, 500))

    def want(section):
        return not args.case or args.case in section

    def emit(name, ms, nbytes, extra):
        mean, med = ms
        gbs = nbytes / (mean / 1e3) / 1e9
        line = {"suite": name, "unit": "GB/s", "value": round(gbs, 2),
                "frac_of_hbm_peak": round(gbs / peak, 4), "peak": peak,
                "peak_kind": f"{peak_kind} HBM copy bandwidth", "us_mean": round(mean * 1e3, 2),
                "us_median": round(med * 1e3, 2), "bytes": int(nbytes), "launches_timed": iters,
                "l2": _L2Flush.DESCRIPTION}
        line.update(extra)
        print(json.dumps(line), flush=True)

    def decode_case(name, w, partition_size=0, extra=None, fp8=False, append=False):
        t = _dev_workload(w, dev)
        L = int(w.seq_lens.max())
        out = torch.empty((w.B, w.Hq, w.d), dtype=torch.bfloat16, device=dev)
        ws = pkv.new_workspace(pkv.decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.d, w.bs, L,
                                                          partition_size), dev)

        def fn(kc=t["kc"], vc=t["vc"]):
            if append:  # every request appends one token: one new row per request
                pkv.paged_attention_decode_append(t["q"], t["kn"], t["vn"], kc, vc, t["bt"],
                                                  t["sl"], w.bs, w.scale, out, max_seq_len=L,
                                                  workspace=ws, partition_size=partition_size)
                return
            pkv.paged_attention_decode(t["q"], kc, vc, t["bt"], t["sl"], w.bs,
                                       w.scale, out, max_seq_len=L, workspace=ws,
                                       partition_size=partition_size, k_scale=t["ks"],
                                       v_scale=t["vs"])
        ms = _time_graph(fn, iters, flush)
        assert pkv.get_device_error() == 0
        # back to back: graphs of B2B_RUN launches over B2B_POOLS copies of the
        # caches (more than L2 holds), events around each graph
        pools = [(t["kc"], t["vc"])] + [(t["kc"].clone(), t["vc"].clone())
                                        for _ in range(B2B_POOLS - 1)]
        b2b = _time_back_to_back(lambda i: fn(*pools[i % B2B_POOLS]), B2B_RUN, 10)
        del pools
        assert pkv.get_device_error() == 0
        e_kv = 1 if fp8 else 2
        nbytes = (2 * int(w.seq_lens.astype(np.int64).sum()) * w.Hkv * w.d * e_kv
                  + w.B * w.Hq * w.d * 4)
        if append:
            nbytes += write_bytes(w.B, w.Hkv, w.d)
        info = {"B": w.B, "Hq": w.Hq, "Hkv": w.Hkv, "d": w.d, "block_size": w.bs,
                "kv_dtype": "fp8_e4m3" if fp8 else "bf16", "partition_size": partition_size,
                "context_tokens": int(w.seq_lens.astype(np.int64).sum()),
                "us_back_to_back": round(b2b * 1e3, 2),
                "GBps_back_to_back": round(nbytes / (b2b / 1e3) / 1e9, 1),
                "back_to_back": f"graphs of {B2B_RUN} launches over {B2B_POOLS} copies of "
                                "the caches, median per launch"}
        info.update(extra or {})
        emit(name, ms, nbytes, info)
        del t, ws, out
        torch.cuda.empty_cache()

    # the 4k workload: permuted pool (as benched) and identity tables (the
    # indirection's cost is the difference)
    if want("gqa_4k"):
        decode_case("decode gqa_4k permuted pool", workloads.gqa_4k(poison=False))
        w = workloads.make_paged([4096] * 16, Hq=32, Hkv=8, d=128, bs=16, dtype="bf16",
                                 seed=1002, poison=False, permute=False, name="gqa_4k_identity")
        decode_case("decode gqa_4k identity tables", w)
    if want("append"):
        decode_case("decode gqa_4k with the fused append (paged_attention_decode_append)",
                    workloads.gqa_4k(poison=False), append=True)
    if want("fp8"):
        decode_case("decode gqa_4k fp8 e4m3 cache", workloads.gqa_4k_fp8(poison=False), fp8=True)
    if want("mixed"):
        decode_case("decode mixed (256 requests, log-uniform 16..8192)",
                    workloads.mixed(poison=False))
    if want("long_ctx"):
        for bs in (8, 16, 32):
            wl = workloads.long_ctx(bs=bs, poison=False)
            for P in (0, 512, 1024, 2048, 4096):
                decode_case(f"decode long_ctx 2 x 131072 bs {bs} partition {P or 'auto'}", wl,
                            partition_size=P)
            del wl
    if want("small_blocks"):
        # block sizes 4 and 2: tensor-core decode fed by one bulk copy per
        # (block, K or V) (blocks of fewer than 8 rows cannot be
        # 128-byte-swizzled TMA boxes)
        for bs in (4, 2):
            w = workloads.make_paged([4096] * 16, Hq=32, Hkv=8, d=128, bs=bs, dtype="bf16",
                                     seed=1002, poison=False, name=f"gqa_4k_bs{bs}")
            decode_case(f"decode 4k batch, block {bs} (row copies)", w)
            del w
    if want("prefix"):
        _suite_prefix(pkv, torch, workloads, dev, iters, flush, emit)
    if want("cache_ops"):
        _suite_cache_ops(pkv, torch, workloads, dev, iters, flush, emit)


# ---------------------------------------------------------------------------
# per-workload section of the headline line: every workload of the scope
# table, each timed on the GPU and with the oracle timed beside it
# ---------------------------------------------------------------------------

def _oracle_rate(w, nthreads: int, budget_s: float, lib, per_head: bool) -> dict:
    """KV GB/s of the oracle on a bounded sample of workload ``w``: whole
    requests (all heads; ``per_head`` False), or one kv head's query group of a
    request at a time (``per_head`` True, for the single-thread figure), taken
    in order until about ``budget_s`` seconds of oracle time.  Bytes are counted
    by the same formula as the GPU (K+V once per kv head + q + out)."""
    import oracle
    G = w.Hq // w.Hkv
    e_kv = w.elem_bytes
    e_q = 4 if w.dtype == "f32" else 2
    ks = None if w.k_scale is None else w.k_scale
    vs = None if w.v_scale is None else w.v_scale
    t_all, nbytes, units = 0.0, 0, 0
    sliced = {}
    order = [b for b in range(w.B) if int(w.seq_lens[b]) > 0]
    heads = range(w.Hkv) if per_head else [None]
    # in order, starting over while the budget lasts (a tiny workload is
    # repeated until the sample is long enough to time)
    order = [order[i % len(order)] for i in range(len(order) * 10_000)] if order else []
    for b in order:
        L = int(w.seq_lens[b])
        for g in heads:
            if g is None:
                q, kc, vc, hk, kss, vss = w.q[b:b + 1], w.k_cache, w.v_cache, w.Hkv, ks, vs
            else:
                if g not in sliced:
                    sliced[g] = (np.ascontiguousarray(w.k_cache[:, g:g + 1]),
                                 np.ascontiguousarray(w.v_cache[:, g:g + 1]))
                kc, vc = sliced[g]
                q = np.ascontiguousarray(w.q[b:b + 1, g * G:(g + 1) * G])
                hk = 1
                kss = None if ks is None else ks[g:g + 1]
                vss = None if vs is None else vs[g:g + 1]
            t0 = time.perf_counter()
            oracle.decode(q, kc, vc, w.block_tables[b:b + 1], w.seq_lens[b:b + 1], w.scale,
                          k_scale=kss, v_scale=vss, nthreads=nthreads, lib=lib)
            t_all += time.perf_counter() - t0
            nbytes += 2 * L * hk * w.d * e_kv + q.shape[1] * w.d * (e_q + e_q)
            units += 1
            if t_all >= budget_s:
                break
        if t_all >= budget_s:
            break
    what = "kv-head groups" if per_head else "whole requests"
    return {"GBps": round(nbytes / t_all / 1e9, 4), "threads": nthreads,
            "sample": f"{units} {what}, {t_all:.2f} s"}


def run_configs(pkv, torch, dev, peak, peak_kind, with_oracle=True, iters=200,
                oracle_budget_s=0.8) -> list:
    """One compact entry per workload: mean decode time over ``iters`` launches
    (each after the L2 flush of _L2Flush, CUDA events around each), KV GB/s by the
    decode byte model, the fraction of the HBM peak, the same for launches issued
    back to back (``us_back_to_back``: graphs of B2B_RUN launches over B2B_POOLS
    copies of the caches, median per launch), and the oracle's KV GB/s on a
    bounded sample of the same workload on all host cores and on one thread.
    """
    import oracle
    import workloads
    flush = _L2Flush(dev)
    lib = oracle.load() if with_oracle else None
    allc = oracle_all_cores(lib) if with_oracle else 0
    entries = []

    def oracle_pair(w):
        if not with_oracle:
            return None
        return {"all_cores": _oracle_rate(w, allc, oracle_budget_s, lib, per_head=False),
                "single_thread": _oracle_rate(w, 1, oracle_budget_s, lib, per_head=True)}

    def nbytes_of(w):
        e_q = 4 if w.dtype == "f32" else 2
        return (2 * int(w.seq_lens.astype(np.int64).sum()) * w.Hkv * w.d * w.elem_bytes
                + w.B * w.Hq * w.d * 2 * e_q)

    def entry(name, w, ms, nbytes, extra=None, oracle_w=None, b2b_ms=None):
        mean, med = ms
        gbs = nbytes / (mean / 1e3) / 1e9
        e = {"workload": name, "us_mean": round(mean * 1e3, 2), "us_median": round(med * 1e3, 2),
             "GBps": round(gbs, 1), "frac_of_peak": round(gbs / peak, 4), "bytes": int(nbytes),
             "tokens_per_s": round(w.B / (mean / 1e3), 1)}
        if b2b_ms is not None:
            g2 = nbytes / (b2b_ms / 1e3) / 1e9
            e.update({"us_back_to_back": round(b2b_ms * 1e3, 2), "GBps_back_to_back": round(g2, 1),
                      "frac_back_to_back": round(g2 / peak, 4)})
        e.update(extra or {})
        e["oracle"] = oracle_pair(oracle_w if oracle_w is not None else w)
        entries.append(e)
        print(json.dumps({"config_line": e}), file=sys.stderr, flush=True)

    def decode_fn(t, w, out, ws, partition_size=0):
        L = int(w.seq_lens.max())
        return lambda kc=t["kc"], vc=t["vc"]: pkv.paged_attention_decode(
            t["q"], kc, vc, t["bt"], t["sl"], w.bs, w.scale, out, max_seq_len=L,
            workspace=ws, partition_size=partition_size, k_scale=t["ks"], v_scale=t["vs"])

    def b2b(t, fn):
        """Median per-launch time (ms) of graphs of B2B_RUN launches of fn(kc, vc)
        back to back over B2B_POOLS copies of the caches (more than L2 holds)."""
        pools = [(t["kc"], t["vc"])] + [(t["kc"].clone(), t["vc"].clone())
                                        for _ in range(B2B_POOLS - 1)]
        ms = _time_back_to_back(lambda i: fn(*pools[i % B2B_POOLS]), B2B_RUN, 10)
        del pools
        torch.cuda.empty_cache()
        assert pkv.get_device_error() == 0
        return ms

    def setup(w, partition_size=0):
        t = _dev_workload(w, dev)
        L = int(w.seq_lens.max())
        odt = torch.float32 if w.dtype == "f32" else torch.bfloat16
        out = torch.empty((w.B, w.Hq, w.d), dtype=odt, device=dev)
        ws = pkv.new_workspace(pkv.decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.d, w.bs, L,
                                                          partition_size), dev)
        return t, out, ws

    def write_fn(t, w):
        if w.dtype == "fp8":
            return lambda: pkv.kv_cache_write_fp8(t["kn"], t["vn"], t["sm"], t["kc"], t["vc"],
                                                  t["ks"], t["vs"])
        return lambda: pkv.kv_cache_write(t["kn"], t["vn"], t["sm"], t["kc"], t["vc"])

    torch.cuda.nvtx.range_push("per-workload section")
    # config 1: tiny fp32 (latency-bound; correctness workload)
    w = workloads.tiny_f32(poison=False)
    t, out, ws = setup(w)
    dec = decode_fn(t, w, out, ws)
    wr = write_fn(t, w)
    ms = _time_graph(lambda: (wr(), dec()), iters, flush)
    entry("tiny_f32: 4 requests [1,17,100,200], 4 q / 2 KV heads, d 64, bs 16, fp32 "
          "(append + decode)", w, ms, nbytes_of(w), {"kv_dtype": "f32"})
    del t, out, ws

    # config 2: the 4k batch, permuted pool and identity tables (indirection cost)
    for name, perm in (("gqa_4k permuted pool", True), ("gqa_4k identity tables", False)):
        w = workloads.make_paged([4096] * 16, Hq=32, Hkv=8, d=128, bs=16, dtype="bf16",
                                 seed=1002, poison=False, permute=perm, name=name)
        t, out, ws = setup(w)
        ms = _time_graph(decode_fn(t, w, out, ws), iters, flush)
        entry(f"{name}: 16 x 4096, 32 q / 8 KV heads, d 128, bs 16, bf16 (decode)", w, ms,
              nbytes_of(w), {"kv_dtype": "bf16"}, b2b_ms=b2b(t, decode_fn(t, w, out, ws)))
        del t, out, ws

    # the same batch with an fp8 (e4m3) cache
    w = workloads.gqa_4k_fp8(poison=False)
    t, out, ws = setup(w)
    ms = _time_graph(decode_fn(t, w, out, ws), iters, flush)
    entry("gqa_4k_fp8: 16 x 4096, e4m3 cache with per-kv-head scales (decode; bytes of codes)",
          w, ms, nbytes_of(w), {"kv_dtype": "fp8_e4m3"}, b2b_ms=b2b(t, decode_fn(t, w, out, ws)))
    del t, out, ws

    # config 3: mixed lengths, append + decode
    w = workloads.mixed(poison=False)
    t, out, ws = setup(w)
    dec = decode_fn(t, w, out, ws)
    Lm = int(w.seq_lens.max())

    def dec_append():  # every request appends one token, inside the decode launch
        pkv.paged_attention_decode_append(t["q"], t["kn"], t["vn"], t["kc"], t["vc"], t["bt"],
                                          t["sl"], w.bs, w.scale, out, max_seq_len=Lm,
                                          workspace=ws)
    ms_dec = _time_graph(dec, iters, flush)
    ms_step = _time_graph(dec_append, iters, flush)
    entry("mixed: 256 requests, log-uniform 16..8192 tokens (decode)", w, ms_dec, nbytes_of(w),
          {"kv_dtype": "bf16", "step_us_mean": round(ms_step[0] * 1e3, 2),
           "step": "paged_attention_decode_append (256 new tokens appended in the decode launch)",
           "context_tokens": int(w.seq_lens.astype(np.int64).sum())}, b2b_ms=b2b(t, dec))
    del t, out, ws, w
    torch.cuda.empty_cache()

    # config 4: shared prefix, per-request decode and prefix-aware decode
    w = workloads.prefix_shared(poison=False)
    t, out, ws = setup(w)
    L = int(w.seq_lens.max())
    plen = (w.info["prefix_tokens"] // w.bs) * w.bs
    pfx_of = torch.zeros(w.B, dtype=torch.int32, device=dev)
    pfx_len = torch.tensor([plen], dtype=torch.int32, device=dev)
    ws_p = pkv.new_workspace(pkv.decode_prefix_workspace_bytes(
        w.B, w.Hq, w.Hkv, w.d, w.bs, L, 1, w.B, w.info["prefix_tokens"]), dev)
    dec = decode_fn(t, w, out, ws)

    def dec_p(kc=t["kc"], vc=t["vc"]):
        pkv.paged_attention_decode_prefix(t["q"], kc, vc, t["bt"], t["sl"], pfx_of,
                                          pfx_len, w.bs, w.scale, out, max_seq_len=L,
                                          max_prefix_members=w.B,
                                          max_prefix_len=w.info["prefix_tokens"], workspace=ws_p)

    def fork_append():
        pkv.copy_blocks(t["kc"], t["vc"], t["pairs"])
        pkv.kv_cache_write(t["kn"], t["vn"], t["sm"], t["kc"], t["vc"])
    logical = nbytes_of(w)
    unique_tok = w.info["prefix_tokens"] + sum(w.info["suffix"])
    unique = 2 * unique_tok * w.Hkv * w.d * 2 + w.B * w.Hq * w.d * 4
    ms_a = _time_graph(dec, iters, flush)
    ms_b = _time_graph(dec_p, iters, flush)
    b2b_a, b2b_b = b2b(t, dec), b2b(t, dec_p)
    ms_sa = _time_graph(lambda: (fork_append(), dec()), iters, flush)
    ms_sb = _time_graph(lambda: (fork_append(), dec_p()), iters, flush)
    common = {"kv_dtype": "bf16", "bytes_kind": "logical (prefix counted once per request)",
              "unique_bytes": unique}
    entry("prefix: 64 requests sharing a 2040-token prefix, per-request decode", w, ms_a,
          logical, dict(common, unique_GBps=round(unique / (ms_a[0] / 1e3) / 1e9, 1),
                        step_us_mean=round(ms_sa[0] * 1e3, 2),
                        step="copy_blocks (64 forks) + kv_cache_write (suffixes) + decode"),
          b2b_ms=b2b_a)
    entry("prefix: the same, prefix-aware decode (shared blocks read once per group)", w, ms_b,
          logical, dict(common, unique_GBps=round(unique / (ms_b[0] / 1e3) / 1e9, 1),
                        step_us_mean=round(ms_sb[0] * 1e3, 2),
                        step="copy_blocks (64 forks) + kv_cache_write (suffixes) + "
                             "paged_attention_decode_prefix"), b2b_ms=b2b_b)
    del t, out, ws, ws_p, w
    torch.cuda.empty_cache()

    # config 5: long context, block sizes 8 / 16 / 32, automatic split
    for bs in (8, 16, 32):
        w = workloads.long_ctx(bs=bs, poison=False)
        t, out, ws = setup(w)
        ms = _time_graph(decode_fn(t, w, out, ws), max(50, iters // 4), flush)
        entry(f"long_ctx: 2 x 131072 tokens, 64 q / 8 KV heads, d 128, bs {bs}, automatic "
              f"split (decode)", w, ms, nbytes_of(w), {"kv_dtype": "bf16", "block_size": bs},
              b2b_ms=b2b(t, decode_fn(t, w, out, ws)))
        del t, out, ws, w
        torch.cuda.empty_cache()
    torch.cuda.nvtx.range_pop()
    assert pkv.get_device_error() == 0
    return entries


def _suite_prefix(pkv, torch, workloads, dev, iters, flush, emit):

    # shared prefix: the step (fork copy + suffix append + decode)
    w = workloads.prefix_shared(poison=False)
    t = _dev_workload(w, dev)
    L = int(w.seq_lens.max())
    out = torch.empty((w.B, w.Hq, w.d), dtype=torch.bfloat16, device=dev)
    ws = pkv.new_workspace(pkv.decode_workspace_bytes(w.B, w.Hq, w.Hkv, w.d, w.bs, L, 0), dev)
    kc0, vc0 = t["kc"].clone(), t["vc"].clone()

    def prefix_step():
        pkv.copy_blocks(t["kc"], t["vc"], t["pairs"])
        pkv.kv_cache_write(t["kn"], t["vn"], t["sm"], t["kc"], t["vc"])
        pkv.paged_attention_decode(t["q"], t["kc"], t["vc"], t["bt"], t["sl"], w.bs, w.scale,
                                   out, max_seq_len=L, workspace=ws)
    ms = _time_graph(prefix_step, iters, flush)
    logical = 2 * int(w.seq_lens.astype(np.int64).sum()) * w.Hkv * w.d * 2 + w.B * w.Hq * w.d * 4
    unique_tok = w.info["prefix_tokens"] + sum(w.info["suffix"])
    unique = 2 * unique_tok * w.Hkv * w.d * 2 + w.B * w.Hq * w.d * 4
    emit("step prefix (64 requests sharing a 2040-token prefix)", ms, logical,
         {"bytes_kind": "logical (prefix counted once per request)", "unique_bytes": unique,
          "unique_GBps": round(unique / (ms[0] / 1e3) / 1e9, 2),
          "step": "copy_blocks (64 forks) + kv_cache_write (suffixes) + decode"})
    # the same step with the shared blocks read once for the group
    pfx_of = torch.zeros(w.B, dtype=torch.int32, device=dev)
    pfx_len = torch.tensor([(w.info["prefix_tokens"] // w.bs) * w.bs], dtype=torch.int32,
                           device=dev)
    ws_p = pkv.new_workspace(pkv.decode_prefix_workspace_bytes(
        w.B, w.Hq, w.Hkv, w.d, w.bs, L, 1, w.B, w.info["prefix_tokens"]), dev)

    def prefix_decode():
        pkv.paged_attention_decode_prefix(t["q"], t["kc"], t["vc"], t["bt"], t["sl"], pfx_of,
                                          pfx_len, w.bs, w.scale, out, max_seq_len=L,
                                          max_prefix_members=w.B,
                                          max_prefix_len=w.info["prefix_tokens"],
                                          workspace=ws_p)

    def prefix_step_shared():
        pkv.copy_blocks(t["kc"], t["vc"], t["pairs"])
        pkv.kv_cache_write(t["kn"], t["vn"], t["sm"], t["kc"], t["vc"])
        prefix_decode()
    ms = _time_graph(prefix_step_shared, iters, flush)
    emit("step prefix, prefix-aware decode (shared blocks read once per group)", ms, logical,
         {"bytes_kind": "logical (prefix counted once per request)", "unique_bytes": unique,
          "unique_GBps": round(unique / (ms[0] / 1e3) / 1e9, 2),
          "step": "copy_blocks (64 forks) + kv_cache_write (suffixes) + "
                  "paged_attention_decode_prefix"})
    ms = _time_graph(lambda: pkv.paged_attention_decode(
        t["q"], t["kc"], t["vc"], t["bt"], t["sl"], w.bs, w.scale, out, max_seq_len=L,
        workspace=ws), iters, flush)
    emit("decode prefix workload, per-request decode", ms, logical,
         {"bytes_kind": "logical", "unique_bytes": unique,
          "unique_GBps": round(unique / (ms[0] / 1e3) / 1e9, 2)})
    ms = _time_graph(prefix_decode, iters, flush)
    emit("decode prefix workload, prefix-aware decode", ms, logical,
         {"bytes_kind": "logical", "unique_bytes": unique,
          "unique_GBps": round(unique / (ms[0] / 1e3) / 1e9, 2)})
    assert pkv.get_device_error() == 0
    del ws_p
    del t, ws, out, kc0, vc0
    torch.cuda.empty_cache()


def _suite_cache_ops(pkv, torch, workloads, dev, iters, flush, emit):
    # cache operations alone
    w = workloads.gqa_4k(poison=False)
    t = _dev_workload(w, dev)
    NB = w.num_blocks
    blk_bytes = 2 * w.Hkv * w.bs * w.d * 2  # K + V of one block
    T = 16384
    rng = np.random.default_rng(7)
    slots = torch.from_numpy(rng.permutation(NB * w.bs)[:T].astype(np.int64)).to(dev)
    kn = torch.randn((T, w.Hkv, w.d), device=dev).to(torch.bfloat16)
    vn = torch.randn((T, w.Hkv, w.d), device=dev).to(torch.bfloat16)
    ms = _time_graph(lambda: pkv.kv_cache_write(kn, vn, slots, t["kc"], t["vc"]), iters, flush)
    emit("kv_cache_write 16384 scattered tokens", ms, 2 * 2 * T * w.Hkv * w.d * 2,
         {"bytes_kind": "read new K,V + write cache rows"})
    ms = _time_graph(lambda: pkv.kv_cache_write(t["kn"], t["vn"], t["sm"], t["kc"], t["vc"]),
                     iters, flush)
    emit("kv_cache_write 16 tokens (one decode step)", ms, 2 * 2 * 16 * w.Hkv * w.d * 2,
         {"bytes_kind": "read new K,V + write cache rows", "note": "launch-latency bound"})
    perm = rng.permutation(NB)
    pairs = torch.from_numpy(np.stack([perm[:1024], perm[1024:2048]], 1).astype(np.int64)).to(dev)
    ms = _time_graph(lambda: pkv.copy_blocks(t["kc"], t["vc"], pairs), iters, flush)
    emit("copy_blocks 1024 pairs", ms, 2 * 1024 * blk_bytes,
         {"bytes_kind": "read + write K and V of each pair"})
    nsw = 1024
    hk = torch.empty((nsw, w.Hkv, w.bs, w.d), dtype=torch.bfloat16).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    out_pairs = torch.from_numpy(np.stack([perm[:nsw], np.arange(nsw)], 1).astype(np.int64)).to(dev)
    in_pairs = torch.from_numpy(np.stack([np.arange(nsw), perm[2048:2048 + nsw]], 1)
                                .astype(np.int64)).to(dev)
    ms = _time_graph(lambda: pkv.swap_blocks(t["kc"], t["vc"], hk, hv, out_pairs), iters, flush)
    emit("swap_blocks device -> pinned host, 1024 blocks", ms, nsw * blk_bytes,
         {"bytes_kind": "K and V bytes moved", "note": "host link bound, not HBM"})
    ms = _time_graph(lambda: pkv.swap_blocks(hk, hv, t["kc"], t["vc"], in_pairs), iters, flush)
    emit("swap_blocks pinned host -> device, 1024 blocks", ms, nsw * blk_bytes,
         {"bytes_kind": "K and V bytes moved", "note": "host link bound, not HBM"})
    assert pkv.get_device_error() == 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-workload section (every workload of the scope table, "
                         "each with the oracle timed beside it)")
    ap.add_argument("--clocks-csv", default="",
                    help="where to keep the raw nvidia-smi samples of the timed region "
                         "(default: a temporary file; the JSON line carries the summary)")
    ap.add_argument("--no-check", action="store_true",
                    help="accepted for older command lines; parity is checked by the tests, "
                         "not by the bench")
    ap.add_argument("--plumbing-only", action="store_true",
                    help="set up the ranks, pass the barriers and the max-over-ranks "
                         "exchange, print n_gpus, and stop (no GPU work; runs on CPU)")
    ap.add_argument("--suite", action="store_true",
                    help="one line per workload of the scope table instead of the headline")
    ap.add_argument("--case", default="",
                    help="with --suite: only the sections whose name contains this "
                         "(gqa_4k, fp8, mixed, long_ctx, small_blocks, prefix, cache_ops)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.impl == "reference":
        # The oracle runs on the host of rank 0 only; other ranks have no work
        # and leave without joining a process group.
        if int(os.environ.get("RANK", "0")) == 0:
            run_reference(args, 0, int(os.environ.get("WORLD_SIZE", "1")))
        return
    if args.suite:
        run_suite(args)
        return
    if args.gpus > 1 and "WORLD_SIZE" not in os.environ:
        sys.exit(relaunch_under_torchrun(args.gpus, sys.argv[1:]))
    rank, world, local = dist_setup(args.gpus)
    if args.plumbing_only:
        # the rank set-up, barriers and max-over-ranks exchange alone (no GPU
        # work): what the multi-rank launch does before and after timing
        try:
            dist_barrier(world)
            top = dist_max(float(rank), world)
            if rank == 0:
                print(json.dumps({"plumbing_only": True, "n_gpus": world, "max_rank": top}),
                      flush=True)
            dist_barrier(world)
        finally:
            dist_done(world)
        return
    try:
        run_ours(args, rank, world, local)
    finally:
        dist_barrier(world)
        dist_done(world)


if __name__ == "__main__":
    main()
