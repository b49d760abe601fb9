"""Hybrid-Block decode benchmark (HySparse2 Cross-Decoder block on B200).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

One step = one decode step of a Hybrid Block: the full-attention layer with
token selection (hs2_full_attn_select) followed by three sparse-attention
layers (hs2_sparse_attn), each with its own query, all reading the same
shared KV cache and the same index list.  The default workload is 256K-token
decode: batch 4, 4 KV heads, GQA 8, head_dim 128, bf16 paged KV (page 64).

Prints one JSON line (rank 0).  Under torchrun every rank runs its own replica
(weak scaling, no data-path collective); the step time is the max over ranks.
"""
from __future__ import annotations

import argparse
import ctypes
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from long_context_decode_full_b200 import synth  # noqa: E402

METRIC = "Hybrid-Block decode steps/s at 256K ctx; achieved HBM GB/s vs B200 peak"
DEFAULT_WORKLOAD = "ctx256k_b4_bf16_paged"
ES = {"f32": 4, "bf16": 2, "e4m3": 1}


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal (about 8 TB/s)


def same_run_copy_peak(dev, nbytes=2 << 30, repeats=6):
    """HBM copy bandwidth measured in this process with the library's own copy
    kernel (hs2_copy_peak): `nbytes` read + `nbytes` written per launch, best
    of `repeats` launches timed with CUDA events.  Returns GB/s and details."""
    from long_context_decode_full_b200 import hs2

    src = torch.empty(nbytes, dtype=torch.uint8, device=dev)
    dst = torch.empty_like(src)
    src.fill_(1)
    stream = torch.cuda.current_stream()
    hs2.copy_peak(dst, src)
    times = []
    for _ in range(repeats):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        hs2.copy_peak(dst, src)
        b.record(stream)
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    del src, dst
    torch.cuda.empty_cache()
    best = min(times)
    gbs = 2.0 * nbytes / (best * 1e-3) / 1e9
    return {"gbs": gbs, "bytes_per_launch": 2 * nbytes, "best_ms": best, "repeats": repeats,
            "what": "hs2_copy_peak: device-to-device copy of %d MiB (read + write), best of %d launches"
                    % (nbytes >> 20, repeats)}


def fracs(achieved_gbs, measured, same_run):
    """The same achieved bandwidth against the three peaks, each labelled."""
    return {"of_measured_peaks_json": achieved_gbs / measured,
            "of_same_run_copy": None if same_run is None else achieved_gbs / same_run,
            "of_nominal_8000_gbs": achieved_gbs / NOMINAL_HBM_GBS}


def algorithmic_bytes(w: synth.Workload):
    """Compulsory bytes of one step: the full layer reads every K and V row
    (+ per-token scales for E4M3) once and writes + reads one fp32 group score
    per selectable position; each sparse layer reads its listed rows."""
    s = w.spec
    lens = [int(x) for x in w.seq_lens.cpu()]
    row = 2 * s.head_dim * ES[s.kv_dtype] + (8 if s.kv_dtype == "e4m3" else 0)  # K+V (+2 scales)
    kv = sum(lens) * s.num_kv_heads * row
    scores = sum(max(0, T - s.window) for T in lens if T - s.window > s.k_global) * s.num_kv_heads * 8
    rows = sum(min(T, s.window + s.k_global) for T in lens) * s.num_kv_heads * row
    qo = s.batch * s.num_q_heads * s.head_dim * ES[s.q_dtype] * 2
    return {"full_attention": kv, "full_layer": kv + scores + qo, "sparse_layer": rows + qo,
            "step": kv + scores + qo + s.sparse_layers * (rows + qo)}


ATTN_SOURCES = ("hs2_full_attn.cu", "hs2_warp_attn.cuh", "hs2_common.cuh")


def _code_only(text: str) -> str:
    """C/C++ source without comments and blank-space runs (a comment edit is
    not a kernel change)."""
    import re
    out, i, n = [], 0, len(text)
    while i < n:
        if text.startswith("//", i):
            j = text.find("\n", i)
            i = n if j < 0 else j
        elif text.startswith("/*", i):
            j = text.find("*/", i + 2)
            i = n if j < 0 else j + 2
        elif text[i] == '"':  # string literal (inline PTX): kept verbatim
            j = i + 1
            while j < n and text[j] != '"':
                j += 2 if text[j] == "\\" else 1
            out.append(text[i:j + 1])
            i = j + 1
        else:
            out.append(text[i])
            i += 1
    return re.sub(r"\s+", " ", "".join(out)).strip()


def attention_source_hash():
    """SHA-256 of the attention kernel's sources, comments and spacing removed."""
    h = hashlib.sha256()
    for name in ATTN_SOURCES:
        with open(os.path.join(ROOT, "long_context_decode_full_b200", "csrc", name)) as f:
            h.update(_code_only(f.read()).encode())
    return h.hexdigest()


def measured_traffic(workload):
    """DRAM bytes (read + write) of one attention launch from the committed ncu
    capture, or None when there is none for this workload or the kernel's
    sources changed since it was taken."""
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(tpath):
        return None
    with open(tpath) as f:
        t = json.load(f)
    if t.get("kernel_source_sha256") != attention_source_hash():
        return None
    return t.get("bytes_per_launch", {}).get(workload)


class Clocks:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.file = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)

    def start(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100"],
                                         stdout=self.file, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        self.proc.wait()
        self.file.seek(0)
        rows = [r.split(",") for r in self.file.read().strip().splitlines() if r.strip()]
        os.unlink(self.file.name)
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            try:
                sm.append(float(r[1]))
                smax = float(r[2])
            except (ValueError, IndexError):
                continue
            for n, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm)}


def setup_dist(gpus: int):
    """One process per GPU (torchrun environment); NCCL on GPUs, gloo on a
    host without one (the CPU tests of the multi-process path)."""
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    cuda = torch.cuda.is_available()
    if world > 1:
        import datetime
        timeout = datetime.timedelta(seconds=120)
        if cuda:
            torch.cuda.set_device(local)
            torch.distributed.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            torch.distributed.init_process_group("gloo", timeout=timeout)
    elif cuda:
        torch.cuda.set_device(0)
    return rank, world, local


def barrier(world):
    if world > 1:
        torch.distributed.barrier()


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    dev = "cuda" if torch.distributed.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], device=dev, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


# ------------------------------------------------------------------ oracle
def oracle_unit_seconds(w: synth.Workload, b: int, kvh: int):
    """Time the CPU oracle on one (sequence, kv head) of the workload: the full
    layer + selection, then every sparse layer.  Returns (seconds, threads)."""
    import numpy as np

    import oracle

    oracle.build()
    s = w.spec
    T = int(w.seq_lens[b])
    slots = synth.slots_of(w, b, torch.arange(T, device=w.k.device))
    G = s.group
    code = {"f32": 0, "bf16": 1, "e4m3": 2}
    k = synth.raw(w.k[slots, kvh:kvh + 1])
    v = synth.raw(w.v[slots, kvh:kvh + 1])
    ks = synth.raw(None if w.k_scale is None else w.k_scale[slots, kvh:kvh + 1])
    vs = synth.raw(None if w.v_scale is None else w.v_scale[slots, kvh:kvh + 1])
    qf = synth.raw(w.q_full[b:b + 1, kvh * G:(kvh + 1) * G])
    qs = [synth.raw(w.q_sparse[l, b:b + 1, kvh * G:(kvh + 1) * G]) for l in range(s.sparse_layers)]
    t0 = time.perf_counter()
    r = oracle.full_attn_select(qf, code[s.q_dtype], k, v, code[s.kv_dtype], np.array([T], np.int32), None, T,
                                s.window, s.k_global, k_scale=ks, v_scale=vs)
    for q in qs:
        oracle.sparse_attn(q, code[s.q_dtype], k, v, code[s.kv_dtype], r["idx"], k_scale=ks, v_scale=vs)
    return time.perf_counter() - t0, 1


def host_cpu():
    """Model name and logical core count of the host running the oracle."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return {"model": model, "nproc": os.cpu_count()}


def workload_config(w: synth.Workload, world: int):
    s = w.spec
    return {"workload": s.name, "batch": s.batch, "seq_len": s.seq_len, "num_kv_heads": s.num_kv_heads,
            "gqa_group": s.group, "head_dim": s.head_dim, "kv_dtype": s.kv_dtype, "page_size": s.page_size,
            "sparse_layers": s.sparse_layers, "window": s.window, "k_global": s.k_global,
            "parallelism": f"replicas x{world}",
            "l2": "inputs larger than L2: %.2f GB of K/V read per step, no flush"
                  % (algorithmic_bytes(w)["full_attention"] / 1e9)}


def cpu_baseline(w: synth.Workload, seconds: float = 10.0, max_units: int = 256):
    """Oracle steps/s from timed (sequence, kv head) units, cycling over the
    step's units until about `seconds` of oracle time has been measured."""
    s = w.spec
    total_units = s.batch * s.num_kv_heads
    secs, n, threads = 0.0, 0, 1
    while n < max_units and (secs < seconds or n == 0):
        b, kvh = divmod(n % total_units, s.num_kv_heads)
        t, threads = oracle_unit_seconds(w, b, kvh)
        secs += t
        n += 1
    per_step = secs / n * total_units
    return {"value": 1.0 / per_step, "unit": "steps/s", "cores": threads, "kind": "oracle",
            "cpu": host_cpu(),
            "sample": f"{n} unit evaluations cycling over the {total_units} (sequence, kv head) units of one step "
                      f"(full layer + selection + {s.sparse_layers} sparse layers), fp64 single-threaded C; "
                      f"step time = mean unit time x {total_units}", "seconds_measured": secs}


# ------------------------------------------------------------------ KV Bridging append
BRIDGE_D_MODEL = 4096  # the pages give no hidden size; a synthetic stand-in


def bridge_bytes(batch, d_model, num_kv_heads, head_dim, elt, scales):
    """Compulsory bytes of one KV Bridging append: both bf16 weight matrices
    once, the bf16 hidden states, and the stored K and V rows (+ their fp32
    scales for E4M3)."""
    n = num_kv_heads * head_dim
    return (2 * d_model * n * 2 + batch * d_model * 2 + 2 * batch * n * elt
            + (2 * batch * num_kv_heads * 4 if scales else 0))


def time_kv_bridge(w, dev, stream, peak, iters=20):
    """The decode-time KV Bridging append on the workload's batch and cache,
    L2 flushed before every launch so the weights come from HBM as they do
    inside a real step.  Two figures:
      - in a graph: a CUDA graph of `iters` x (L2 flush, append) minus a
        graph of `iters` flushes, per append -- its cost inside a captured
        decode step, without per-launch host overhead (the reported one);
      - isolated: each launch between its own pair of CUDA events, queued
        behind a device-side sleep so the host's call overhead is not in the
        interval; it includes the launch's own latency.
    It writes the rows at position T_b - 1, so it runs after every other
    measurement."""
    from long_context_decode_full_b200 import hs2

    s = w.spec
    N = s.num_kv_heads * s.head_dim
    g = torch.Generator(device=dev).manual_seed(1234)
    h = torch.randn(s.batch, BRIDGE_D_MODEL, device=dev, generator=g).to(torch.bfloat16)
    wk = (torch.randn(BRIDGE_D_MODEL, N, device=dev, generator=g) * 0.02).to(torch.bfloat16)
    wv = (torch.randn(BRIDGE_D_MODEL, N, device=dev, generator=g) * 0.02).to(torch.bfloat16)
    ws = torch.zeros(hs2.kv_bridge_workspace_bytes(s.batch, BRIDGE_D_MODEL, s.num_kv_heads, s.head_dim),
                     dtype=torch.uint8, device=dev)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)

    def call():
        hs2.kv_bridge_append(h, wk, wv, w.k, w.v, w.seq_lens, w.page_table, w.page_size, w.k_scale, w.v_scale,
                             workspace=ws)

    for _ in range(3):
        call()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(iters)]
    torch.cuda.synchronize()
    torch.cuda._sleep(50_000_000)  # the host queues every launch before the GPU reaches the first
    for a, b in ev:
        flush.zero_()
        a.record(stream)
        call()
        b.record(stream)
    torch.cuda.synchronize()
    isolated_us = statistics.mean(a.elapsed_time(b) for a, b in ev) * 1e3

    def graph_ms(body):
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            for _ in range(iters):
                body()
        gr.replay()
        torch.cuda.synchronize()
        t = []
        for _ in range(5):
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            gr.replay()
            b.record()
            torch.cuda.synchronize()
            t.append(a.elapsed_time(b))
        del gr
        return statistics.median(t)

    def flush_and_call():
        flush.zero_()
        call()

    try:
        graph_us = (graph_ms(flush_and_call) - graph_ms(flush.zero_)) / iters * 1e3
        method = f"CUDA graph of {iters} x (L2 flush, append) minus a graph of {iters} flushes"
        us = graph_us
    except RuntimeError as e:  # capture unavailable: the isolated figure stands
        graph_us, us = None, isolated_us
        method = f"isolated launches (graph capture failed: {str(e).splitlines()[0][:120]})"
    torch.cuda.synchronize()
    nbytes = bridge_bytes(s.batch, BRIDGE_D_MODEL, s.num_kv_heads, s.head_dim, w.k.element_size(),
                          w.k_scale is not None)
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"d_model": BRIDGE_D_MODEL, "us": us, "method": method, "graph_us": graph_us,
            "isolated_launch_us": isolated_us, "algorithmic_bytes": nbytes, "achieved_gbs": gbs,
            "frac": gbs / peak, "roofline_us": nbytes / (peak * 1e3), "launches": 1,
            "l2": "flushed before each launch",
            "what": "k = h W_k, v = h W_v for the new token of every sequence, stored at position T_b - 1 "
                    "(E4M3: per-(token, kv head) scale); bytes = both weight matrices + hidden + stored rows"}


# ------------------------------------------------------------------ block-level selection
def time_block_selection(w, ws, out, idx, stream, block=16, iters=50):
    """The full layer with the first-generation block-level selection in
    place of the token-level one (the comparator), on the same inputs: mean
    time of `iters` back-to-back calls, and of the same number of token-level
    calls for reference (both CUDA events around the whole run)."""
    from long_context_decode_full_b200 import hs2

    s = w.spec
    if s.k_global % block:
        return None

    def run(fn):
        for _ in range(3):
            fn()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        a.record(stream)
        for _ in range(iters):
            fn()
        b.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(b) / iters

    blk = run(lambda: hs2.full_attn_select_blocks(w.q_full, w.k, w.v, w.seq_lens, w.page_table, w.page_size,
                                                  s.window, s.k_global, block, w.k_scale, w.v_scale, out=out,
                                                  idx_out=idx, workspace=ws))
    tok = run(lambda: hs2.full_attn_select(w.q_full, w.k, w.v, w.seq_lens, w.page_table, w.page_size, s.window,
                                           s.k_global, w.k_scale, w.v_scale, out=out, idx_out=idx, workspace=ws))
    return {"block": block, "full_layer_ms_block_selection": blk, "full_layer_ms_token_selection": tok,
            "calls": iters, "what": "full layer (attention + selection) per call, back to back, CUDA events"}


# ------------------------------------------------------------------ GPU arm
def run_gpu(args, rank, world, local):
    from long_context_decode_full_b200 import hs2

    spec = synth.WORKLOADS[args.workload]
    if args.seq_len:
        spec = spec.replace(seq_len=args.seq_len)
    if args.kv_heads:
        spec = spec.replace(num_kv_heads=args.kv_heads)
    if args.batch:
        spec = spec.replace(batch=args.batch)
    w = synth.generate(spec, seed=args.seed + rank, device="cuda")
    s = spec
    dev = torch.device("cuda", local)
    outs = [torch.empty_like(w.q_full) for _ in range(1 + s.sparse_layers)]
    idx = torch.empty(s.batch, s.num_kv_heads, s.window + s.k_global, dtype=torch.int32, device=dev)
    ws = hs2.alloc_workspace(s.batch, s.num_kv_heads, s.group, s.head_dim, w.t_cap, dev)
    stream = torch.cuda.current_stream()
    K, W = args.steps, args.warmup
    KB = max(3, min(K, 200))  # steps of the per-kernel breakdown (after the timed region)
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(KB)]

    def step(e=None):
        # the marked breakdown steps run the separate kernels (their boundary carries the event)
        hs2.full_attn_select(w.q_full, w.k, w.v, w.seq_lens, w.page_table, w.page_size, s.window, s.k_global,
                             w.k_scale, w.v_scale, out=outs[0], idx_out=idx, workspace=ws,
                             mark_event=None if e is None else e[1], fused=args.fused and e is None)
        if e is not None:
            e[2].record(stream)
        for l in range(s.sparse_layers):
            hs2.sparse_attn(w.q_sparse[l], w.k, w.v, idx, w.k_scale, w.v_scale, w.page_size, out=outs[1 + l])

    copy = same_run_copy_peak(dev) if not args.no_copy_peak else None
    for e in ev:  # materialise the event handles before the first marked call
        for x in e:
            x.record(stream)
    for _ in range(W):
        step()
    torch.cuda.synchronize()
    if hs2.workspace_status(ws) != 0:
        raise RuntimeError("device-side wait expired during warm-up: " + hs2.last_error())

    clocks = Clocks(local)
    barrier(world)
    torch.cuda.synchronize()
    clocks.start()
    time.sleep(0.3)
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for i in range(K):  # plain steps: no event between two kernels of the timed region
        step()
    t_end.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    barrier(world)
    ms_total = t_start.elapsed_time(t_end)
    ms_total = max_over_ranks(ms_total, world)
    ms_step = ms_total / K
    # per-kernel breakdown on separate steps: events after the attention kernel
    # and after the selection (they serialise those kernel boundaries, so these
    # steps are not the timed ones)
    for i in range(KB):
        ev[i][0].record(stream)
        step(ev[i])
    torch.cuda.synchronize()
    attn_ms = statistics.mean(ev[i][0].elapsed_time(ev[i][1]) for i in range(KB))
    sel_ms = statistics.mean(ev[i][1].elapsed_time(ev[i][2]) for i in range(KB))
    marked_ms = statistics.mean(ev[i][0].elapsed_time(ev[i + 1][0]) for i in range(KB - 1))

    # e2e: queries in from pinned host memory, outputs + index list back, every step.
    # The step's inputs travel in one pinned buffer and its results in one device
    # buffer (one copy each way); the kernels read and write views of them.
    def packed(tensors, device):
        offs, n = [], 0
        for t in tensors:
            offs.append(n)
            n += (t.numel() * t.element_size() + 255) // 256 * 256
        buf = torch.empty(n, dtype=torch.uint8, device=device)
        views = [buf[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape) for o, t in zip(offs, tensors)]
        return buf, views

    ins = [w.q_full] + [w.q_sparse[l] for l in range(s.sparse_layers)] + [w.seq_lens]
    in_dev, in_views = packed(ins, dev)
    in_host = torch.empty_like(in_dev, device="cpu").pin_memory()
    off = 0
    for t in ins:  # the inputs laid out in the pinned buffer as in the device one
        nb = t.numel() * t.element_size()
        in_host[off:off + nb].view(t.dtype).view(t.shape).copy_(t.cpu())
        off += (nb + 255) // 256 * 256
    q_dev, lens_dev = in_views[:-1], in_views[-1]
    out_dev, out_views = packed(outs + [idx], dev)
    outs_e2e, idx_e2e = out_views[:-1], out_views[-1]
    out_host = torch.empty_like(out_dev, device="cpu").pin_memory()
    h2d = in_host.numel()
    d2h = out_host.numel()
    K2 = max(3, min(K, args.e2e_steps))

    # Through the C ABI as a C caller makes it: the cache, query and output
    # descriptors are built once (their buffers do not move), then every step
    # calls hs2_full_attn_select and hs2_sparse_attn with them.
    L = hs2.lib()
    kc, vc = hs2.cache_desc(w.k, w.k_scale, w.page_size), hs2.cache_desc(w.v, w.v_scale, w.page_size)
    qds = [hs2.heads_desc(q) for q in q_dev]
    ods = [hs2.heads_desc(o) for o in outs_e2e]
    sp_ = hs2._stream(None)
    max_pages = 1 if w.page_table is None else w.page_table.shape[1]
    full_fn = L.hs2_full_attn_select_fused if args.fused else L.hs2_full_attn_select
    full_args = (ctypes.byref(qds[0]), ctypes.byref(kc), ctypes.byref(vc), hs2._ptr(lens_dev), hs2._ptr(w.page_table),
                 max_pages, s.window, s.k_global, ctypes.byref(ods[0]), hs2._ptr(idx_e2e), hs2._ptr(ws), ws.numel(), sp_)
    sparse_args = [(ctypes.byref(qds[1 + l]), ctypes.byref(kc), ctypes.byref(vc), hs2._ptr(idx_e2e),
                    s.window + s.k_global, ctypes.byref(ods[1 + l]), sp_) for l in range(s.sparse_layers)]

    def e2e_step():
        in_dev.copy_(in_host, non_blocking=True)
        rc = full_fn(*full_args)
        for a in sparse_args:
            rc |= L.hs2_sparse_attn(*a)
        if rc:
            raise RuntimeError("C call failed: " + hs2.last_error())
        out_host.copy_(out_dev, non_blocking=True)
        torch.cuda.current_stream().synchronize()

    for _ in range(3):
        e2e_step()
    barrier(world)
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a0.record(stream)
    for _ in range(K2):
        e2e_step()
    a1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(a0.elapsed_time(a1), world) / K2
    status = hs2.workspace_status(ws)

    ab = algorithmic_bytes(w)
    peak, peak_kind = peaks()
    copy_gbs = None if copy is None else copy["gbs"]
    attn_gbs = ab["full_attention"] / (attn_ms * 1e-3) / 1e9
    step_gbs = ab["step"] / (ms_step * 1e-3) / 1e9
    traffic = measured_traffic(args.workload)
    res = {
        "metric": METRIC,
        "value": world * 1000.0 / ms_step,
        "unit": "steps/s",
        "n_gpus": world,
        "steps": K,
        "warmup": W,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": {"bf16": "bf16", "e4m3": "e4m3", "f32": "f32"}[s.kv_dtype],
        "data": "synthetic",
        "config": dict(workload_config(w, world), full_layer_call="fused" if args.fused else "separate kernels"),
        "roofline": {"bound": "hbm", "kernel": "full_attn_mma_kernel", "achieved": attn_gbs, "peak": peak,
                     "unit": "GB/s", "frac": attn_gbs / peak, "traffic": traffic,
                     "peak_source": f"{peak_kind} copy bandwidth (MEASURED_PEAKS.json hbm_gbs)",
                     "fracs": fracs(attn_gbs, peak, copy_gbs),
                     "algorithmic_bytes_per_launch": ab["full_attention"], "kernel_ms": attn_ms},
        "step_roofline": {"achieved": step_gbs, "frac": step_gbs / peak, "fracs": fracs(step_gbs, peak, copy_gbs),
                          "compulsory_bytes": ab["step"],
                          "roofline_steps_per_s": peak * 1e9 / ab["step"],
                          "roofline_steps_per_s_same_run_copy": None if copy_gbs is None else copy_gbs * 1e9 / ab["step"],
                          "roofline_steps_per_s_nominal": NOMINAL_HBM_GBS * 1e9 / ab["step"],
                          "selection_ms": sel_ms, "sparse_and_rest_ms": marked_ms - attn_ms - sel_ms,
                          "breakdown": f"{KB} separate steps with events after the attention kernel and after the "
                                       f"selection ({marked_ms:.4f} ms/step with those events)"},
        "copy_peak_same_run": copy,
        "nominal_hbm_gbs": NOMINAL_HBM_GBS,
        "e2e": {"value": world * 1000.0 / e2e_ms, "unit": "steps/s", "h2d_bytes_per_step": h2d,
                "d2h_bytes_per_step": d2h, "steps": K2,
                "what": "through the C ABI (hs2_full_attn_select, hs2_sparse_attn; descriptors built once): "
                        "queries and lengths copied in from one pinned host buffer, outputs and index list copied "
                        "out as one buffer and synced, every step; the KV cache stays resident"},
        "gpu_launches": K * ((3 if args.fused else 4) + s.sparse_layers),
        "clocks": clk,
        "device_status": status,
    }
    if world == 1 and not args.no_block_timing:
        res["block_selection"] = time_block_selection(w, ws, outs[0], idx, stream)
    if not args.no_bridge and world == 1:
        # a per-GPU figure; with one process there is no NCCL thread about
        # while the graph is captured
        res["kv_bridge_append"] = time_kv_bridge(w, dev, stream, peak)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    return res


def run_reference(args, rank, world, local):
    """The oracle as it stands, timed on the host cores (rank 0 only).  One
    step is the whole decode step: every (sequence, kv head) unit through the
    full layer, the selection and every sparse layer, one after another on one
    core; `--warmup` untimed steps, then `--steps` timed ones."""
    if rank != 0:
        return None
    spec = synth.WORKLOADS[args.workload]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    w = synth.generate(spec, seed=args.seed, device=dev)
    units = [divmod(n, spec.num_kv_heads) for n in range(spec.batch * spec.num_kv_heads)]
    times = []
    for i in range(args.warmup + args.steps):
        t = 0.0
        for b, kvh in units:
            dt, threads = oracle_unit_seconds(w, b, kvh)
            t += dt
        if i >= args.warmup:
            times.append(t)
    ms = statistics.mean(times) * 1000.0
    v = 1000.0 / ms
    return {"metric": METRIC, "value": v, "unit": "steps/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
            "config": dict(workload_config(w, world), full_layer_call="fused" if args.fused else "separate kernels"),
            "cpu_baseline": {"value": v, "unit": "steps/s", "cores": threads, "kind": "oracle", "cpu": host_cpu(),
                             "sample": f"whole steps: all {len(units)} (sequence, kv head) units of the workload, "
                                       f"each through the full layer, the selection and {spec.sparse_layers} sparse "
                                       "layers (fp64, single-threaded C); the time counts the oracle calls only, "
                                       "not the gathering of each unit's rows into host memory"},
            "e2e": {"value": v, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(synth.WORKLOADS))
    ap.add_argument("--no-bridge", action="store_true", help="skip the KV Bridging append measurement")
    ap.add_argument("--impl", default="hs2", choices=["hs2", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--e2e-steps", type=int, default=500)
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="oracle time for the CPU baseline sample")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-copy-peak", action="store_true", help="skip the same-run copy-bandwidth measurement")
    ap.add_argument("--no-block-timing", action="store_true", help="skip the block-level selection timing")
    ap.add_argument("--fused", action="store_true",
                    help="time the fused full-layer call (attention + score pass in one persistent kernel)")
    ap.add_argument("--seq-len", type=int, default=0, help="override the workload's context (profiling runs)")
    ap.add_argument("--kv-heads", type=int, default=0, help="override the workload's KV heads (experiments)")
    ap.add_argument("--batch", type=int, default=0, help="override the workload's batch (experiments)")
    args = ap.parse_args()
    if args.impl == "reference":
        rank = int(os.environ.get("RANK", "0"))
        res = run_reference(args, rank, int(os.environ.get("WORLD_SIZE", "1")), 0)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    rank, world, local = setup_dist(args.gpus)
    try:
        res = run_gpu(args, rank, world, local)
        if rank == 0:
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
