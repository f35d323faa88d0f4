#!/usr/bin/env python
"""Benchmark of the kv2d hot path on synthetic long-context inputs.

One step = one pass of the whole path over one batch: kv2d_compress of the
prompt (window statistics, scoring passes, channel top-c, segment selection,
budget, packing), kv2d_append of one new token per (sequence, KV head), and
kv2d_decode_attn of every query head over the compressed cache plus its dense
tail.  The compressed-cache bookkeeping is reset at the start of each step so
every step compresses the full prompt again.

Default workload: one Llama-3-8B-shaped attention layer (32 query / 8 KV
heads, d = 128), batch 1, 32K-token context in fp16, segment 64, window 64,
budget 20%.  Inputs are resident in HBM (K + V = 134 MB > the 126 MB L2) and
L2 is flushed between timed steps by writing a 256 MB buffer.

Prints ONE JSON line (rank 0).  Multi-GPU: one process per GPU (torchrun);
each rank compresses and decodes its own independent batch (weak scaling, no
data-path collective); the reported time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "decode-attn us/step & HBM GB/s over compressed KV; kv2d_compress GB/s"
UNIT = "GB/s"
DEFAULT_WORKLOAD = "llama3_8b_32k"
SMI_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")


def rank_seed(seed, rank):
    """Seed of a rank's batch: every rank draws its own independent batch
    (weak scaling: per-GPU work is fixed as the number of ranks grows)."""
    return seed + 1000 * rank


def max_over_ranks(x, dist, device):
    """The largest x over all ranks (a job takes as long as its slowest
    rank); x itself without a process group."""
    if dist is None:
        return x
    import torch
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(bytes_per_rank, world, ms_per_step):
    """Whole-job GB/s: the bytes all ranks processed over the slowest rank's
    time per step."""
    return bytes_per_rank * world / (ms_per_step * 1e-3) / 1e9


def profiled_traffic(kernel, workload):
    """DRAM bytes (read + write) per launch of `kernel` on `workload` from the
    committed ncu summary profiles/<kernel>_<workload>.md, or None when there
    is none or the kernel's source file has changed since the capture (the
    summary records the SHA-256 of the source it was measured with)."""
    import hashlib
    root = os.path.dirname(os.path.abspath(__file__))
    path = os.path.join(root, "profiles", f"{kernel}_{workload}.md")
    if not os.path.exists(path):
        return None
    fields = {}
    with open(path) as f:
        for line in f:
            if ":" in line and line.split(":", 1)[0] in ("traffic_bytes_per_launch", "kernel_source",
                                                        "kernel_source_sha256"):
                k, v = line.split(":", 1)
                fields[k] = v.strip()
    try:
        with open(os.path.join(root, fields["kernel_source"]), "rb") as f:
            sha = hashlib.sha256(f.read()).hexdigest()
        if sha != fields["kernel_source_sha256"]:
            return None
        return int(fields["traffic_bytes_per_launch"])
    except (KeyError, OSError, ValueError):
        return None


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["kv2d", "reference"], default="kv2d")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true",
                    help="skip the CUDA-graph decode timing and the budget-1 decode")
    ap.add_argument("--no-decode-large", action="store_true",
                    help="skip the decode-only measurement on the batch-16 x 128K cache")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0)), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def dense_bytes(wl, lens):
    return sum(int(T) for T in lens) * wl.num_kv_heads * wl.head_dim * 2 * 2


# ------------------------------------------------------------------ clocks


class ClockSampler:
    def __init__(self, gpu_index):
        self.proc = None
        self.gpu = gpu_index

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={SMI_FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-i", str(self.gpu)],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.lines = []
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out = ""
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        sm, mx, reasons = [], 0, set()
        names = ["active", "hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown",
                 "sw_power_cap"]
        for ln in getattr(self, "lines", []):
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = max(mx, float(parts[2]))
            except ValueError:
                continue
            for nm, val in zip(names[1:], parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(nm)
        load = [s for s in sm if s > 0.5 * mx] if mx else sm
        return {"sm_mhz": statistics.median(load) if load else None,
                "sm_max_mhz": mx or None, "reasons": sorted(reasons), "samples": len(sm)}


# --------------------------------------------------------------- reference


def run_reference(args, rank):
    """The reference arm: the fp64 CPU oracle, as it stands, on host cores,
    each step a bounded sample of the workload (units in parallel threads)."""
    if rank != 0:
        return
    import numpy as np
    import torch
    from kv_cache_compression_kv2d_b200 import synth
    from oracle import oracle as O
    O.build()
    wl = synth.WORKLOADS[args.workload]
    lens = synth.lengths(wl, args.seed)
    ncpu = os.cpu_count() or 1
    threads = max(1, min(ncpu, 2))
    batch = synth.generate(wl.with_(batch=1, seq_len=int(lens[0]), ragged_min=0,
                                    num_kv_heads=threads), seed=args.seed)
    p = O.params(wl.head_dim, wl.group, wl.segment_len, wl.window, wl.r, wl.c,
                 float(np.float32(wl.budget)), float(np.float32(1 / np.sqrt(wl.head_dim))))
    T = int(batch.seq_len[0])
    G = wl.group

    def unit(h):
        K = batch.k[0, h, :T].numpy()
        V = batch.v[0, h, :T].numpy()
        qw = batch.qw[0, h * G:(h + 1) * G].reshape(-1, wl.head_dim).numpy()
        res = O.compress_unit(p, T, 0, K, V, qw)
        nc = res["nseg"] * wl.segment_len
        O.decode_unit(p, res["arena"], res["offs"], res["strat"], K[nc:], V[nc:],
                      batch.q[0, h * G:(h + 1) * G].numpy())

    times = []
    for i in range(args.warmup + args.steps):
        t0 = time.perf_counter()
        O.parallel_map(unit, list(range(threads)), threads=threads)
        dt = time.perf_counter() - t0
        if i >= args.warmup:
            times.append(dt)
    sample_bytes = T * threads * wl.head_dim * 4
    ms = 1e3 * statistics.mean(times)
    value = sample_bytes / (ms * 1e-3) / 1e9
    sample = (f"{threads} of {wl.batch * wl.num_kv_heads} (sequence, KV head) units of "
              f"{wl.name}: compress of {T} tokens + one decode each, per step")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic",
            "config": {"workload": wl.name, "global_batch": wl.batch, "seq_len": T,
                       "parallelism": "host threads", "l2": "n/a (CPU)"},
            "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def cpu_baseline(wl, batch_host, p_gpu, budget_s=30.0):
    """The oracle as it stands, on the host cores, over a bounded sample of
    units of the same workload (one thread per unit)."""
    import numpy as np
    from oracle import oracle as O
    O.build()
    ncpu = os.cpu_count() or 1
    units = [(b, h) for b in range(wl.batch) for h in range(wl.num_kv_heads)]
    n = max(1, min(len(units), ncpu))
    units = units[:n]
    p = O.params(wl.head_dim, wl.group, wl.segment_len, wl.window, wl.r, wl.c,
                 float(np.float32(wl.budget)), float(np.float32(p_gpu.scale)))
    G = wl.group

    def unit(bh):
        b, h = bh
        T = int(batch_host.seq_len[b])
        K = batch_host.k[b, h, :T].numpy()
        V = batch_host.v[b, h, :T].numpy()
        qw = batch_host.qw[b, h * G:(h + 1) * G].reshape(-1, wl.head_dim).numpy()
        res = O.compress_unit(p, T, 0, K, V, qw)
        nc = res["nseg"] * wl.segment_len
        O.decode_unit(p, res["arena"], res["offs"], res["strat"], K[nc:], V[nc:],
                      batch_host.q[b, h * G:(h + 1) * G].numpy())
        return T

    t0 = time.perf_counter()
    toks = O.parallel_map(unit, units, threads=n)
    dt = time.perf_counter() - t0
    nbytes = sum(toks) * wl.head_dim * 4
    model = None
    try:
        with open("/proc/cpuinfo") as f:
            model = next((l.split(":", 1)[1].strip() for l in f if l.startswith("model name")), None)
    except OSError:
        pass
    return {"value": nbytes / dt / 1e9, "unit": UNIT, "cores": n, "kind": "oracle", "cpu_model": model,
            "sample": f"{n} of {wl.batch * wl.num_kv_heads} (sequence, KV head) units "
                      f"(compress + one decode each) in {dt:.1f} s"}


# ------------------------------------------------------------------- kv2d


def decode_batch16_128k(B, synth, torch, dev, stream, hbm, steps):
    """Decode alone over the batch-16 x 128K cache (8 KV heads, four-class
    segment mix, budget 15 %): 1.29 GB of packed bytes, larger than L2, a size
    at which decode is bound by HBM rather than by its fixed phases."""
    wl = synth.WORKLOADS["llama3_8b_b16_128k_mix"]
    bt = synth.generate(wl, seed=0, device=dev, extra_capacity=16)
    lens = [int(x) for x in bt.seq_len]
    scale = float(torch.tensor(1.0 / wl.head_dim ** 0.5, dtype=torch.float32))
    p = B.params(wl.head_dim, wl.num_q_heads, wl.num_kv_heads, wl.segment_len, wl.window, wl.r,
                 wl.c, wl.budget, scale)
    dv = B.dense(bt.k, bt.v)
    cc = B.CompressedCache(p, wl.batch, bt.capacity, device=dev)
    ws_c = B.workspace(B.kv2d_workspace_bytes(p, B.OP_COMPRESS, wl.batch, max(lens)), dev)
    ws_d = B.workspace(B.kv2d_workspace_bytes(p, B.OP_DECODE, wl.batch, bt.capacity), dev)
    B.kv2d_compress(p, wl.batch, lens, [0] * wl.batch, dv, bt.qw, cc.struct, ws_c, stream=stream)
    seq = torch.tensor(lens, dtype=torch.int32, device=dev)
    out = torch.empty((wl.batch, wl.num_q_heads, wl.head_dim), dtype=torch.float16, device=dev)

    def decode():
        B.kv2d_decode_attn(p, wl.batch, cc.struct, dv, seq, bt.capacity, bt.q, out, ws_d, stream=stream)

    for _ in range(3):
        decode()
    evs = []
    for _ in range(steps):
        a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        decode()
        b_.record(stream)
        evs.append((a, b_))
    torch.cuda.synchronize(dev)
    assert B.kv2d_read_status(ws_c, stream) == 0 and B.kv2d_read_status(ws_d, stream) == 0
    us = 1e3 * statistics.mean(a.elapsed_time(b_) for a, b_ in evs)
    ce = cc.comp_end.cpu().tolist()
    tail = sum((lens[b] - ce[b]) * wl.num_kv_heads for b in range(wl.batch))
    nbytes = (int(cc.used_bytes.sum()) + 8 * int(cc.n_segs.sum()) + tail * wl.head_dim * 4 +
              2 * wl.batch * wl.num_q_heads * wl.head_dim * 2)
    del bt, dv, cc, ws_c, ws_d, out
    torch.cuda.empty_cache()
    gbs = nbytes / (us * 1e-6) / 1e9
    return {"workload": wl.name, "us_per_call": us, "bytes_per_call": nbytes, "hbm_gbs": gbs,
            "hbm_frac": gbs / hbm, "calls": steps,
            "l2": "no flush: 1.29 GB of packed bytes per call > L2"}


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return

    import torch
    torch.cuda.set_device(local)
    dist = None
    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))

    from kv_cache_compression_kv2d_b200 import binding as B
    from kv_cache_compression_kv2d_b200 import build as kbuild
    from kv_cache_compression_kv2d_b200 import synth
    kbuild.build()
    B.lib()

    wl = synth.WORKLOADS[args.workload]
    dev = torch.device("cuda", local)
    host = synth.generate(wl, seed=rank_seed(args.seed, rank), device="cpu", extra_capacity=16)
    lens = [int(x) for x in host.seq_len]
    k = host.k.to(dev)
    v = host.v.to(dev)
    qw = host.qw.to(dev)
    q = host.q.to(dev)
    bt = host.block_table.to(dev) if host.block_table is not None else None
    scale = float(torch.tensor(1.0 / wl.head_dim ** 0.5, dtype=torch.float32))
    p = B.params(wl.head_dim, wl.num_q_heads, wl.num_kv_heads, wl.segment_len, wl.window, wl.r,
                 wl.c, wl.budget, scale)
    dv = B.dense(k, v, bt, wl.block_size) if bt is not None else B.dense(k, v)
    cap = host.capacity
    cc = B.CompressedCache(p, wl.batch, cap, device=dev)
    ws_c = B.workspace(B.kv2d_workspace_bytes(p, B.OP_COMPRESS, wl.batch, max(lens)), dev)
    ws_d = B.workspace(B.kv2d_workspace_bytes(p, B.OP_DECODE, wl.batch, cap), dev)
    ws_a = B.workspace(256, dev)
    kn, vn, _ = synth.decode_tokens(wl, 0, seed=args.seed, device=dev, mu=host.mu.to(dev))
    out = torch.empty((wl.batch, wl.num_q_heads, wl.head_dim), dtype=torch.float16, device=dev)
    seq0 = torch.tensor(lens, dtype=torch.int32, device=dev)
    seq = seq0.clone()
    zeros_ce = [0] * wl.batch
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)   # 256 MB > L2
    stream = torch.cuda.current_stream(dev)

    def reset():
        cc.reset()
        seq.copy_(seq0)

    def compress():
        B.kv2d_compress(p, wl.batch, lens, zeros_ce, dv, qw, cc.struct, ws_c, stream=stream)

    def append():
        B.kv2d_append(p, wl.batch, dv, kn, vn, seq, ws_a, stream=stream)

    def decode():
        B.kv2d_decode_attn(p, wl.batch, cc.struct, dv, seq, cap, q, out, ws_d, stream=stream)

    def step():
        reset()
        compress()
        append()
        decode()

    gpu_index = local
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if local < len(ids):
            gpu_index = ids[local]

    def barrier():
        torch.cuda.synchronize(dev)
        if dist is not None:
            dist.barrier()

    with ClockSampler(gpu_index) as clk:
        # warm-up: W steps, then keep the GPU busy ~1 s so clocks settle
        for _ in range(max(3, args.warmup)):
            step()
        torch.cuda.synchronize(dev)
        t_end = time.time() + 1.0
        while time.time() < t_end:
            step()
            torch.cuda.synchronize(dev)
        assert B.kv2d_read_status(ws_c, stream) == 0 and B.kv2d_read_status(ws_d, stream) == 0

        # ---- timed region: exactly K steps, L2 flushed between steps
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        barrier()
        for i in range(args.steps):
            flush.zero_()
            ev[i][0].record(stream)
            step()
            ev[i][1].record(stream)
        barrier()
        step_ms = [a.elapsed_time(b) for a, b in ev]

        # ---- per-kernel CUDA-event times: the same K steps again with the
        # library's profiler on (its event records sit between launches and
        # stop consecutive kernels from overlapping, so the headline step
        # time above is taken without them)
        B.kv2d_profile_enable(True)
        for i in range(args.steps):
            flush.zero_()
            step()
        torch.cuda.synchronize(dev)
        B.kv2d_profile_enable(False)
        prof = B.kv2d_profile_read()

        # ---- decode alone and compress alone (L2 flushed before each)
        dec_ms, comp_ms = [], []
        for i in range(args.steps):
            flush.zero_()
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            decode()
            b_.record(stream)
            dec_ms.append((a, b_))
        for i in range(args.steps):
            reset()
            flush.zero_()
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            compress()
            b_.record(stream)
            comp_ms.append((a, b_))
        torch.cuda.synchronize(dev)
        dec_ms = [a.elapsed_time(b_) for a, b_ in dec_ms]
        comp_ms = [a.elapsed_time(b_) for a, b_ in comp_ms]

        # ---- 100 back-to-back decodes captured in one CUDA graph (launch
        # overhead amortised; the 32K cache then stays in L2 between calls)
        graph_us = None
        if not args.no_graph:
            try:
                g_stream = torch.cuda.Stream(dev)
                g_stream.wait_stream(stream)
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph, stream=g_stream):
                    for _ in range(100):
                        B.kv2d_decode_attn(p, wl.batch, cc.struct, dv, seq, cap, q, out, ws_d,
                                           stream=g_stream)
                stream.wait_stream(g_stream)
                graph.replay()
                torch.cuda.synchronize(dev)
                a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                for _ in range(5):
                    graph.replay()
                b_.record(stream)
                torch.cuda.synchronize(dev)
                graph_us = 1e3 * a.elapsed_time(b_) / 500
                del graph
            except RuntimeError as exc:   # reported, not fatal: the step numbers stand
                graph_us = f"capture failed: {exc}"[:200]

        # ---- the same prompt compressed at budget 1 (every segment FULL):
        # decode over the uncompressed cache, for the speedup of the packed one
        dense_dec_us = None
        if not args.no_graph:
            p1 = B.params(wl.head_dim, wl.num_q_heads, wl.num_kv_heads, wl.segment_len, wl.window,
                          wl.r, wl.c, 1.0, scale)
            cc1 = B.CompressedCache(p1, wl.batch, cap, device=dev)
            B.kv2d_compress(p1, wl.batch, lens, zeros_ce, dv, qw, cc1.struct, ws_c, stream=stream)
            ev1 = []
            for i in range(args.steps + 3):
                flush.zero_()
                a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                a.record(stream)
                B.kv2d_decode_attn(p1, wl.batch, cc1.struct, dv, seq, cap, q, out, ws_d, stream=stream)
                b_.record(stream)
                if i >= 3:
                    ev1.append((a, b_))
            torch.cuda.synchronize(dev)
            dense_dec_us = 1e3 * statistics.mean(a.elapsed_time(b_) for a, b_ in ev1)
            del cc1
        # leave the cache in its post-step state for the byte accounting
        step()
        torch.cuda.synchronize(dev)
    assert B.kv2d_read_status(ws_c, stream) == 0 and B.kv2d_read_status(ws_d, stream) == 0

    total_ms = max_over_ranks(sum(step_ms), dist, dev)
    ms_step = total_ms / args.steps
    nbytes = dense_bytes(wl, lens)
    value = job_throughput(nbytes, world, ms_step)

    # ---- algorithmic work per launch
    hbm, tf_burst, tf_sust, src = peaks()
    used = cc.used_bytes.cpu().tolist()
    nsegs = cc.n_segs.cpu().tolist()
    ce = cc.comp_end.cpu().tolist()
    seq_after = seq.cpu().tolist()
    tail_tokens = sum((seq_after[b] - ce[b]) * wl.num_kv_heads for b in range(wl.batch))
    dec_bytes = (sum(used) + 8 * sum(nsegs) + tail_tokens * wl.head_dim * 4 +
                 2 * wl.batch * wl.num_q_heads * wl.head_dim * 2)
    dec_us = 1e3 * statistics.mean(dec_ms)
    comp_us = 1e3 * statistics.mean(comp_ms)
    flops_pass = 2.0 * wl.num_q_heads * wl.window * sum(lens) * wl.head_dim
    seg_tokens = sum((T // wl.segment_len) * wl.segment_len for T in lens)
    kv_seg_bytes = seg_tokens * wl.num_kv_heads * wl.head_dim * 2
    work = {
        "score_pass1": ("tensor", flops_pass),
        "score_pass2": ("tensor", 2.0 * wl.num_q_heads * wl.window * seg_tokens * wl.head_dim),
        # K rows in; a 16-byte keep mask and the fp64 g_t out per token
        "chan_topc": ("hbm", kv_seg_bytes + seg_tokens * wl.num_kv_heads * (16 + 8)),
        "pack": ("hbm", 2 * sum(used)),   # gathers about as many bytes as it writes
        "decode": ("hbm", dec_bytes),
    }
    kernels = {}
    for name, (tot, n) in prof.items():
        if n:
            kernels[name] = {"launches": n, "avg_us": 1e3 * tot / n,
                             "share": tot / max(sum(t for t, _ in prof.values()), 1e-12)}
    dominant = max(kernels, key=lambda k_: kernels[k_]["avg_us"] * kernels[k_]["launches"])
    kind, amount = work.get(dominant, ("hbm", 0.0))
    avg_s = kernels[dominant]["avg_us"] * 1e-6
    if kind == "tensor":
        achieved = amount / avg_s / 1e12
        roof = {"bound": "tensor", "achieved": achieved, "peak": tf_burst, "unit": "TFLOP/s",
                "frac": achieved / tf_burst, "traffic": profiled_traffic(dominant, wl.name),
                "kernel": dominant, "peak_source": f"{src} bf16 burst (fp16 runs at the bf16 rate)"}
    else:
        achieved = amount / avg_s / 1e9
        roof = {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
                "frac": achieved / hbm, "traffic": profiled_traffic(dominant, wl.name),
                "kernel": dominant,
                "peak_source": f"{src} HBM copy"}
    gpu_launches = sum(v_["launches"] for v_ in kernels.values())
    # the scoring contraction, both passes (executed MMA flops = algorithmic)
    scoring = None
    if "score_pass1" in kernels and "score_pass2" in kernels:
        t12 = (kernels["score_pass1"]["avg_us"] + kernels["score_pass2"]["avg_us"]) * 1e-6
        sflops = flops_pass + work["score_pass2"][1]
        scoring = {"tflops": sflops / t12 / 1e12, "frac": sflops / t12 / 1e12 / tf_burst,
                   "peak": tf_burst, "peak_source": f"{src} bf16 burst"}
    # compress, algorithmic bytes: K and V of the region read once, the window
    # queries, the packed bytes written, and s (4 B) and g (8 B) per token
    comp_alg = (nbytes + wl.batch * wl.num_q_heads * wl.window * wl.head_dim * 2 + sum(used) +
                seg_tokens * wl.num_kv_heads * 12)

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        hk = host.k.pin_memory()
        hv = host.v.pin_memory()
        hqw = host.qw.pin_memory()
        hq = host.q.pin_memory()
        hkn, hvn = kn.cpu().pin_memory(), vn.cpu().pin_memory()
        hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in (hk, hv, hqw, hq, hkn, hvn))
        if bt is not None:
            hbt = host.block_table.pin_memory()
            h2d += hbt.numel() * 4
        d2h = hout.numel() * hout.element_size()
        evs = []
        for i in range(max(3, args.warmup) + args.steps):
            a, b_ = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(stream)
            k.copy_(hk, non_blocking=True)
            v.copy_(hv, non_blocking=True)
            qw.copy_(hqw, non_blocking=True)
            q.copy_(hq, non_blocking=True)
            kn.copy_(hkn, non_blocking=True)
            vn.copy_(hvn, non_blocking=True)
            if bt is not None:
                bt.copy_(hbt, non_blocking=True)
            step()
            hout.copy_(out, non_blocking=True)
            b_.record(stream)
            if i >= max(3, args.warmup):
                evs.append((a, b_))
        torch.cuda.synchronize(dev)
        e_ms = max_over_ranks(sum(a.elapsed_time(b_) for a, b_ in evs), dist, dev) / args.steps
        e2e = {"value": job_throughput(nbytes, world, e_ms), "unit": UNIT,
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e_ms}

    dec_large = None
    if world == 1 and not args.no_decode_large:
        dec_large = decode_batch16_128k(B, synth, torch, dev, stream, hbm, max(args.steps, 5))

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = cpu_baseline(wl, host, p)

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": {"workload": wl.name, "global_batch": wl.batch * world, "seq_len": max(lens),
                   "num_q_heads": wl.num_q_heads, "num_kv_heads": wl.num_kv_heads,
                   "head_dim": wl.head_dim, "segment_len": wl.segment_len,
                   "window": wl.window, "budget": wl.budget,
                   "parallelism": f"dp{world}" if world > 1 else "single GPU",
                   "l2": "flushed between steps (256 MB write); inputs 134 MB > L2",
                   "value_is": "dense KV bytes (K+V of the prompt) per step / step time"},
        "decode": {"us_per_step": dec_us, "bytes_per_step": dec_bytes,
                   "hbm_gbs": dec_bytes / (dec_us * 1e-6) / 1e9,
                   "hbm_frac": dec_bytes / (dec_us * 1e-6) / 1e9 / hbm,
                   "hbm_frac_of_8tbs_nominal": dec_bytes / (dec_us * 1e-6) / 1e9 / 8000.0,
                   "graph_us_per_call": graph_us,
                   "graph_note": "100 back-to-back calls in one CUDA graph; the cache stays in L2",
                   "budget1_us": dense_dec_us,
                   "speedup_vs_budget1": (dense_dec_us / dec_us) if dense_dec_us else None},
        "compress": {"us": comp_us, "gbs": nbytes / (comp_us * 1e-6) / 1e9,
                     "alg_bytes": comp_alg, "hbm_frac": comp_alg / (comp_us * 1e-6) / 1e9 / hbm},
        "scoring": scoring,
        "decode_batch16_128k": dec_large,
        "kernels": kernels,
        "kernels_note": "per-launch CUDA-event times from a profiled repeat of the K timed steps",
        "roofline": roof,
        "cpu_baseline": cpu,
        "e2e": e2e,
        "gpu_launches": gpu_launches,
        "clocks": clk.summary(),
    }
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
