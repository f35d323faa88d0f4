#!/usr/bin/env python
"""Benchmark of the kv2d hot path on synthetic long-context inputs.

One step = one pass of the whole path over one batch: kv2d_compress of the
prompts (window statistics, scoring passes, channel top-c, segment selection,
budget, packing), kv2d_append of one new token per (sequence, KV head), and
kv2d_decode_attn of every query head over the compressed cache plus its dense
tail.  The compressed-cache bookkeeping is reset at the start of each step so
every step compresses the full prompts again.

Default workload (the largest single-GPU configuration): one
Llama-3-8B-shaped attention layer (32 query / 8 KV heads, d = 128), batch 16
x 128K-token contexts in fp16, segment 64, window 64, budget 15 %, segment
classes mixed so that all four strategies occur.  The dense K + V is 8.6 GB,
far larger than the 126 MB L2, and L2 is also flushed between timed steps.
The other configurations (the 32K layer, the 1M-token layer, the ragged
paged batch of 32 with a periodic re-compression) are timed as extra keys:
compress alone and decode alone.

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
DEFAULT_WORKLOAD = "llama3_8b_b16_128k_mix"
EXTRA_WORKLOADS = ("llama3_8b_32k", "llama3_8b_1m", "ragged32_paged")
SMI_FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
VALUE_IS = "dense KV bytes (K+V of the prompts) per step / step time"


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


def profiled_traffic(kernel, tokens):
    """DRAM bytes (read + write) of one launch of `kernel` over `tokens`
    tokens, from the committed ncu summary profiles/<kernel>_*.md whose
    `kernel_source_sha256` still matches the kernel's source file: the
    captured launch's traffic scaled by tokens (the kernels' traffic grows in
    proportion to the tokens they read).  None when no current summary
    exists.  Returns (bytes, note)."""
    import glob
    import hashlib
    for path in sorted(glob.glob(os.path.join(ROOT, "profiles", f"{kernel}_*.md"))):
        fields = {}
        with open(path) as f:
            for line in f:
                if ":" in line:
                    k, v = line.split(":", 1)
                    if k in ("traffic_bytes_per_launch", "tokens_per_launch", "kernel_source",
                             "kernel_source_sha256", "workload"):
                        fields[k] = v.strip()
        try:
            with open(os.path.join(ROOT, fields["kernel_source"]), "rb") as f:
                sha = hashlib.sha256(f.read()).hexdigest()
            if sha != fields["kernel_source_sha256"]:
                continue
            per = int(fields["traffic_bytes_per_launch"]) / int(fields["tokens_per_launch"])
            note = (f"ncu dram__bytes_read.sum + dram__bytes_write.sum of one launch on "
                    f"{fields.get('workload', '?')} ({os.path.basename(path)}), scaled by tokens")
            return per * tokens, note
        except (KeyError, OSError, ValueError, ZeroDivisionError):
            continue
    return None, "no ncu summary of the current kernel source"


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
    ap.add_argument("--no-extras", action="store_true",
                    help="skip the compress / decode timings of the other configurations")
    return ap.parse_args()


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), float(d.get("bf16_tflops_sustained", 0)), "measured"
    except Exception:
        return 6650.0, 1590.0, 1400.0, "fallback"


def roofline_of(kind, amount, avg_s, hbm, tf_burst, tf_sust, src):
    """Roofline of one kernel: `amount` algorithmic bytes ("hbm") or flops
    ("tensor") per launch over its average launch time `avg_s`.  A tensor
    kernel timed inside the step is held to the sustained bf16 GEMM figure
    (the burst one, or the fallback, when no sustained figure exists), with
    the burst fraction beside it."""
    if kind == "tensor":
        achieved = amount / avg_s / 1e12
        tf_s = tf_sust if tf_sust > 0 else tf_burst
        return {"bound": "tensor", "achieved": achieved, "peak": tf_s, "unit": "TFLOP/s",
                "frac": achieved / tf_s,
                "peak_source": (f"{src} bf16 sustained" if tf_sust > 0 else f"{src} bf16 burst") +
                               " (fp16 runs at the bf16 rate; timed inside the step)",
                "frac_of_burst": achieved / tf_burst}
    achieved = amount / avg_s / 1e9
    return {"bound": "hbm", "achieved": achieved, "peak": hbm, "unit": "GB/s",
            "frac": achieved / hbm, "peak_source": f"{src} HBM copy"}


def scoring_of(flops1, flops2, us1, us2, tf_burst, tf_sust, src):
    """Both scoring passes together (executed MMA flops = algorithmic flops):
    TFLOP/s over the sum of their average launch times, as a fraction of the
    sustained bf16 figure (the passes run inside multi-millisecond steps
    under the power cap) and of the burst figure."""
    t12 = (us1 + us2) * 1e-6
    tflops = (flops1 + flops2) / t12 / 1e12
    tf_s = tf_sust if tf_sust > 0 else tf_burst
    return {"tflops": tflops, "frac": tflops / tf_s, "peak": tf_s,
            "peak_source": f"{src} bf16 sustained" if tf_sust > 0 else f"{src} bf16 burst",
            "frac_of_burst": tflops / tf_burst, "burst_peak": tf_burst,
            "pass1_tflops": flops1 / (us1 * 1e-6) / 1e12, "pass2_tflops": flops2 / (us2 * 1e-6) / 1e12}


def dense_bytes(wl, lens):
    return sum(int(T) for T in lens) * wl.num_kv_heads * wl.head_dim * 2 * 2


def config_of(wl, lens, world):
    """The workload's description, shared by both arms of the benchmark."""
    return {"workload": wl.name, "global_batch": wl.batch * world, "seq_len": max(int(x) for x in lens),
            "num_q_heads": wl.num_q_heads, "num_kv_heads": wl.num_kv_heads,
            "head_dim": wl.head_dim, "segment_len": wl.segment_len, "window": wl.window,
            "budget": wl.budget, "segment_mix": wl.segment_mix,
            "parallelism": f"dp{world}" if world > 1 else "single GPU",
            "l2": "flushed between steps (256 MB write); inputs larger than L2",
            "value_is": VALUE_IS}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            return next((l.split(":", 1)[1].strip() for l in f if l.startswith("model name")), None)
    except OSError:
        return None


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


# ------------------------------------------------------- CPU oracle sample


def cpu_sample_units(wl, seed, n):
    """The seeded sample of (sequence, KV head) units the oracle is timed on
    (both arms use the same sample)."""
    import numpy as np
    units = wl.batch * wl.num_kv_heads
    rng = np.random.default_rng(seed + 424242)
    pick = sorted(rng.choice(units, size=min(n, units), replace=False).tolist())
    return [(u // wl.num_kv_heads, u % wl.num_kv_heads) for u in pick]


def cpu_sample_size():
    """Units in the CPU sample: one per host core, at most 16 (about 10 s of
    oracle work per unit of a 128K-token sequence)."""
    return max(1, min(os.cpu_count() or 1, 16))


def host_units(batch, wl, units):
    """fp16 host copies of the sampled units' prompt rows, window queries and
    decode queries (inputs of the oracle)."""
    out = []
    G = wl.group
    from kv_cache_compression_kv2d_b200 import synth
    for b, h in units:
        T = int(batch.seq_len[b])
        k, v = synth.dense_rows(batch, b, h, 0, T)
        out.append(dict(T=T, K=k.cpu().numpy(), V=v.cpu().numpy(),
                        qw=batch.qw[b, h * G:(h + 1) * G].reshape(-1, wl.head_dim).cpu().numpy(),
                        q=batch.q[b, h * G:(h + 1) * G].cpu().numpy()))
    return out


def oracle_unit_phases(O, p, x):
    """The oracle over one unit, step by step with a clock around each phase:
    scoring (window statistics, lse and s_t), selection (channel top-c and
    g_t, top-r and error proxies per segment, hulls and the budget walk),
    packing (every segment's bytes) and decode (attention of the G heads over
    the packed segments and the dense tail).  Returns the phases' seconds."""
    import numpy as np
    pc = time.perf_counter
    T, S = x["T"], p.S
    nseg = T // S
    t0 = pc()
    Kd = x["K"].astype(np.float64)
    qw = x["qw"].astype(np.float64)
    a = O.win_stats(p, qw)
    _, s = O.score(p, T, 0, Kd, qw)
    t1 = pc()
    cidx, g = O.channel(p, Kd[:nseg * S], a)
    tidx = np.zeros((nseg, p.r), np.uint8)
    E = np.zeros((nseg, 4))
    for j in range(nseg):
        tidx[j] = O.topr(p, s[j * S:(j + 1) * S])
        E[j] = O.segment_errors(p, s[j * S:(j + 1) * S], g[j * S:(j + 1) * S], tidx[j])
    st, strat, used = O.budget(p, E)
    assert st == 0
    t2 = pc()
    parts, offs, off = [], np.zeros(nseg, np.int64), 0
    for j in range(nseg):
        rows = slice(j * S, (j + 1) * S)
        seg = O.pack_segment(p, int(strat[j]), x["K"][rows], x["V"][rows], tidx[j], cidx[rows])
        offs[j] = off
        off += seg.size
        parts.append(seg)
    arena = np.concatenate(parts) if parts else np.zeros(0, np.uint8)
    t3 = pc()
    O.decode_unit(p, arena, offs, strat, x["K"][nseg * S:], x["V"][nseg * S:], x["q"])
    t4 = pc()
    return {"scoring": t1 - t0, "selection": t2 - t1, "packing": t3 - t2, "decode": t4 - t3}


def oracle_sample(wl, xs, scale):
    """The oracle on the sample, one unit per host thread (units are
    independent).  Returns (wall seconds, per-phase thread seconds, dense
    bytes of the sample)."""
    import numpy as np
    from oracle import oracle as O
    O.build()
    p = O.params(wl.head_dim, wl.group, wl.segment_len, wl.window, wl.r, wl.c,
                 float(np.float32(wl.budget)), float(np.float32(scale)))
    t0 = time.perf_counter()
    res = O.parallel_map(lambda x: oracle_unit_phases(O, p, x), xs, threads=len(xs))
    wall = time.perf_counter() - t0
    phases = {k: sum(r[k] for r in res) for k in res[0]}
    nbytes = sum(x["T"] for x in xs) * wl.head_dim * 4
    return wall, phases, nbytes


def cpu_record(wl, units, xs, wall, phases, nbytes):
    total_units = wl.batch * wl.num_kv_heads
    tot = sum(phases.values())
    return {"value": nbytes / wall / 1e9, "unit": UNIT, "cores": len(xs), "kind": "oracle",
            "cpu_model": cpu_model(), "host_cores": os.cpu_count(),
            "sample": (f"{len(xs)} of {total_units} (sequence, KV head) units of {wl.name} "
                       f"(seeded: {units}), each compress of its whole prompt + one decode, one "
                       f"unit per thread, in {wall:.1f} s"),
            "extrapolated_step_s": wall * total_units / len(xs),
            "extrapolation": "linear in the unit count (units are independent): "
                             "sample wall time x all units / sampled units",
            "phase_thread_s": phases,
            "phase_share": {k: v / tot for k, v in phases.items()}}


# --------------------------------------------------------------- reference


def run_reference(args, rank):
    """The reference arm: the fp64 CPU oracle, as it stands, on host cores,
    each step the same bounded sample of the workload as the kv2d arm's
    cpu_baseline (the same units on the same number of threads)."""
    if rank != 0:
        return
    import torch
    from kv_cache_compression_kv2d_b200 import synth
    wl = synth.WORKLOADS[args.workload]
    world = int(os.environ.get("WORLD_SIZE", "1"))
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    batch = synth.generate(wl, seed=rank_seed(args.seed, 0), device=dev, extra_capacity=16)
    lens = [int(x) for x in batch.seq_len]
    units = cpu_sample_units(wl, args.seed, cpu_sample_size())
    xs = host_units(batch, wl, units)
    del batch
    if dev == "cuda":
        torch.cuda.empty_cache()
    scale = float(torch.tensor(1.0 / wl.head_dim ** 0.5, dtype=torch.float32))
    walls, last = [], None
    for i in range(args.warmup + args.steps):
        wall, phases, nbytes = oracle_sample(wl, xs, scale)
        if i >= args.warmup:
            walls.append(wall)
            last = (wall, phases, nbytes)
    ms = 1e3 * statistics.mean(walls)
    value = last[2] / (ms * 1e-3) / 1e9
    cpu = cpu_record(wl, units, xs, ms * 1e-3, last[1], last[2])
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": UNIT,
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(wl, lens, world),
            "cpu_baseline": cpu,
            "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------- kv2d


def decode_bytes(wl, cc, seq):
    """Algorithmic bytes of one decode call: the packed payload used, the
    descriptors, the dense tail's K and V rows, q and out."""
    used = int(cc.used_bytes.sum())
    nsegs = int(cc.n_segs.sum())
    ce = cc.comp_end.cpu().tolist()
    sq = seq.cpu().tolist()
    tail = sum((sq[b] - ce[b]) * wl.num_kv_heads for b in range(wl.batch))
    return used + 8 * nsegs + tail * wl.head_dim * 4 + 2 * wl.batch * wl.num_q_heads * wl.head_dim * 2


def select_bytes(wl, cc, seq):
    """Algorithmic bytes of one selection decode at a rate: every candidate's
    stored key (dense row, or index + value pairs) and descriptor, a 4-byte
    score written and read per candidate slot and a 4-byte index per kept
    slot, the kept candidates' value rows (their keys were read already),
    the dense tail's K and V rows, q and out."""
    import numpy as np
    S, r, c, d = wl.segment_len, wl.r, wl.c, wl.head_dim
    desc = cc.desc.cpu().numpy().view(np.uint64)
    nsg = cc.n_segs.cpu().numpy()
    ce = cc.comp_end.cpu().tolist()
    sq = seq.cpu().tolist()
    key = {0: S * d * 2, 1: r * d * 2, 2: S * c * 3, 3: r * c * 3}
    ntok = {0: S, 1: r, 2: S, 3: r}
    kbytes = slots = 0
    cands = []
    for u in range(desc.shape[0]):
        st = ((desc[u, :nsg[u]] >> np.uint64(32)) & np.uint64(255)).astype(int)
        cnt = np.bincount(st, minlength=4)
        kbytes += sum(int(cnt[k]) * key[k] for k in range(4)) + 8 * int(nsg[u])
        slots += int(nsg[u]) * S
        cands.append((int(nsg[u]) * S, sum(int(cnt[k]) * ntok[k] for k in range(4))))
    tail = sum((sq[b] - ce[b]) * wl.num_kv_heads for b in range(wl.batch))

    def at(rate):
        kept = sum(min(nc, int(np.ceil(np.float64(np.float32(rate)) * ns))) for ns, nc in cands)
        return (kbytes + 8 * slots + 4 * kept + kept * d * 2 + tail * d * 4 +
                2 * wl.batch * wl.num_q_heads * d * 2)
    return at


def compress_alg_bytes(wl, lens, used):
    """Algorithmic bytes of kv2d_compress: K and V of the region read once,
    the window queries, the packed bytes written, and s (4 B) and g (8 B)
    per segment token."""
    seg_tokens = sum((T // wl.segment_len) * wl.segment_len for T in lens)
    return (dense_bytes(wl, lens) + wl.batch * wl.num_q_heads * wl.window * wl.head_dim * 2 + used +
            seg_tokens * wl.num_kv_heads * 12)


def event_pair(torch):
    return torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)


def timed(torch, stream, fn, n, before=None, flush=None):
    """Mean CUDA-event milliseconds of fn() over n calls on stream, each call
    preceded (outside the events) by before() and an L2 flush."""
    evs = []
    for _ in range(n):
        if before is not None:
            before()
        if flush is not None:
            flush.zero_()
        a, b = event_pair(torch)
        a.record(stream)
        fn()
        b.record(stream)
        evs.append((a, b))
    torch.cuda.synchronize()
    return statistics.mean(a.elapsed_time(b) for a, b in evs)


def measure_extra(name, B, synth, torch, dev, stream, flush, hbm, n):
    """Compress alone and decode alone on another configuration (L2 flushed
    before each call); for the ragged paged batch also one periodic
    re-compression of the trailing region after 128 appended tokens."""
    wl = synth.WORKLOADS[name]
    extra = wl.recompress_every + 16 if wl.recompress_every else 16
    bt = synth.generate(wl, seed=0, device=dev, extra_capacity=extra)
    lens = [int(x) for x in bt.seq_len]
    scale = float(torch.tensor(1.0 / wl.head_dim ** 0.5, dtype=torch.float32))
    p = B.params(wl.head_dim, wl.num_q_heads, wl.num_kv_heads, wl.segment_len, wl.window, wl.r,
                 wl.c, wl.budget, scale)
    paged = bt.block_table is not None
    dv = B.dense(bt.k, bt.v, bt.block_table, wl.block_size) if paged else B.dense(bt.k, bt.v)
    cap = bt.capacity
    cc = B.CompressedCache(p, wl.batch, cap, device=dev)
    ws_c = B.workspace(B.kv2d_workspace_bytes(p, B.OP_COMPRESS, wl.batch, max(lens)), dev)
    ws_d = B.workspace(B.kv2d_workspace_bytes(p, B.OP_DECODE, wl.batch, cap), dev)
    zeros = [0] * wl.batch
    seq = torch.tensor(lens, dtype=torch.int32, device=dev)
    out = torch.empty((wl.batch, wl.num_q_heads, wl.head_dim), dtype=torch.float16, device=dev)

    def compress():
        B.kv2d_compress(p, wl.batch, lens, zeros, dv, bt.qw, cc.struct, ws_c, stream=stream)

    def decode():
        B.kv2d_decode_attn(p, wl.batch, cc.struct, dv, seq, cap, bt.q, out, ws_d, stream=stream)

    for _ in range(3):
        cc.reset()
        compress()
    comp_ms = timed(torch, stream, compress, n, before=cc.reset, flush=flush)
    cc.reset()
    compress()
    decode()
    dec_ms = timed(torch, stream, decode, n, flush=flush)
    assert B.kv2d_read_status(ws_c, stream) == 0 and B.kv2d_read_status(ws_d, stream) == 0
    used = int(cc.used_bytes.sum())
    dbytes = decode_bytes(wl, cc, seq)
    calg = compress_alg_bytes(wl, lens, used)
    rec = {"compress": {"us": 1e3 * comp_ms, "gbs": dense_bytes(wl, lens) / (comp_ms * 1e-3) / 1e9,
                        "alg_bytes": calg, "hbm_frac": calg / (comp_ms * 1e-3) / 1e9 / hbm},
           "decode": {"us_per_call": 1e3 * dec_ms, "bytes_per_call": dbytes,
                      "hbm_gbs": dbytes / (dec_ms * 1e-3) / 1e9,
                      "hbm_frac": dbytes / (dec_ms * 1e-3) / 1e9 / hbm},
           "dense_bytes": dense_bytes(wl, lens), "calls": n, "l2": "flushed before each call"}
    if wl.recompress_every:
        # 128 decode steps of appends, then the periodic compression of the
        # complete segments of [comp_end, seq_len); the cache bookkeeping is
        # put back before each timed repeat so every repeat does the same work
        ws_a = B.workspace(256, dev)
        for step in range(wl.recompress_every):
            kn, vn, _ = synth.decode_tokens(wl, step, device=dev, mu=bt.mu)
            B.kv2d_append(p, wl.batch, dv, kn, vn, seq, ws_a, stream=stream)
        torch.cuda.synchronize()
        seq_h = seq.cpu().tolist()
        ce_h = cc.comp_end.cpu().tolist()
        saved = cc.book.clone()

        def recompress():
            B.kv2d_compress(p, wl.batch, seq_h, ce_h, dv, bt.qw, cc.struct, ws_c, stream=stream)

        re_ms = timed(torch, stream, recompress, n, before=lambda: cc.book.copy_(saved), flush=flush)
        region = sum(seq_h[b] - ce_h[b] for b in range(wl.batch))
        assert B.kv2d_read_status(ws_c, stream) == 0 and B.kv2d_read_status(ws_a, stream) == 0
        rec["recompress"] = {"us": 1e3 * re_ms, "region_tokens_per_sequence_mean": region / wl.batch,
                             "note": "compression of [comp_end, seq_len) after 128 appended tokens"}
    del bt, dv, cc, ws_c, ws_d, out
    torch.cuda.empty_cache()
    return rec


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
    stream = torch.cuda.current_stream(dev)
    # inputs are drawn on the device (seeded); host copies serve the
    # end-to-end timing and the CPU baseline
    bat = synth.generate(wl, seed=rank_seed(args.seed, rank), device=dev, extra_capacity=16)
    lens = [int(x) for x in bat.seq_len]
    k, v, qw, q, bt = bat.k, bat.v, bat.qw, bat.q, bat.block_table
    scale = float(torch.tensor(1.0 / wl.head_dim ** 0.5, dtype=torch.float32))
    p = B.params(wl.head_dim, wl.num_q_heads, wl.num_kv_heads, wl.segment_len, wl.window, wl.r,
                 wl.c, wl.budget, scale)
    dv = B.dense(k, v, bt, wl.block_size) if bt is not None else B.dense(k, v)
    cap = bat.capacity
    cc = B.CompressedCache(p, wl.batch, cap, device=dev)
    ws_c = B.workspace(B.kv2d_workspace_bytes(p, B.OP_COMPRESS, wl.batch, max(lens)), dev)
    ws_d = B.workspace(B.kv2d_workspace_bytes(p, B.OP_DECODE, wl.batch, cap), dev)
    ws_a = B.workspace(256, dev)
    kn, vn, _ = synth.decode_tokens(wl, 0, seed=args.seed, device=dev, mu=bat.mu)
    out = torch.empty((wl.batch, wl.num_q_heads, wl.head_dim), dtype=torch.float16, device=dev)
    seq0 = torch.tensor(lens, dtype=torch.int32, device=dev)
    seq = seq0.clone()
    zeros_ce = [0] * wl.batch
    flush = torch.empty(64 * 1024 * 1024, dtype=torch.float32, device=dev)   # 256 MB > L2

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
        ev = [event_pair(torch) for _ in range(args.steps)]
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
        dec_ms = timed(torch, stream, decode, args.steps, flush=flush)
        comp_ms = timed(torch, stream, compress, args.steps, before=reset, flush=flush)

        # ---- 100 back-to-back decodes captured in one CUDA graph (launch
        # overhead amortised)
        graph_us = None
        if not args.no_graph:
            step()
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
                a, b_ = event_pair(torch)
                a.record(stream)
                for _ in range(5):
                    graph.replay()
                b_.record(stream)
                torch.cuda.synchronize(dev)
                graph_us = 1e3 * a.elapsed_time(b_) / 500
                del graph
            except RuntimeError as exc:   # reported, not fatal: the step numbers stand
                graph_us = f"capture failed: {exc}"[:200]

        # ---- the same prompts compressed at budget 1 (every segment FULL):
        # decode over the uncompressed cache, for the speedup of the packed one
        dense_dec_us = None
        if not args.no_graph:
            p1 = B.params(wl.head_dim, wl.num_q_heads, wl.num_kv_heads, wl.segment_len, wl.window,
                          wl.r, wl.c, 1.0, scale)
            cc1 = B.CompressedCache(p1, wl.batch, cap, device=dev)
            B.kv2d_compress(p1, wl.batch, lens, zeros_ce, dv, qw, cc1.struct, ws_c, stream=stream)

            def decode1():
                B.kv2d_decode_attn(p1, wl.batch, cc1.struct, dv, seq, cap, q, out, ws_d, stream=stream)

            decode1()
            dense_dec_us = 1e3 * timed(torch, stream, decode1, args.steps, flush=flush)
            del cc1
            torch.cuda.empty_cache()
        # ---- decode with decode-time token selection at the pages' two
        # rates (6.25 % and 12.5 % of the compressed context), L2 flushed
        step()
        sel_rec = {}
        ws_s = B.workspace(B.kv2d_workspace_bytes(p, B.OP_DECODE_SELECT, wl.batch, cap), dev)
        for rate in (0.0625, 0.125):
            def decode_sel():
                B.kv2d_decode_attn_select(p, wl.batch, cc.struct, dv, seq, cap, q, out, rate, ws_s,
                                          stream=stream)

            decode_sel()
            sel_rec[str(rate)] = {"us_per_call": 1e3 * timed(torch, stream, decode_sel, args.steps,
                                                             flush=flush)}
            B.kv2d_profile_read()
            B.kv2d_profile_enable(True)
            for _ in range(3):
                flush.zero_()
                decode_sel()
            torch.cuda.synchronize(dev)
            B.kv2d_profile_enable(False)
            sel_rec[str(rate)]["kernels_us"] = {k: 1e3 * t / n for k, (t, n) in B.kv2d_profile_read().items()
                                                if n and k.startswith("sel_")}
        assert B.kv2d_read_status(ws_s, stream) == 0
        del ws_s
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
    used = int(cc.used_bytes.sum())
    dec_bytes = decode_bytes(wl, cc, seq)
    dec_us = 1e3 * dec_ms
    comp_us = 1e3 * comp_ms
    sel_bytes = select_bytes(wl, cc, seq)
    for rate, rec in sel_rec.items():
        nb = sel_bytes(float(rate))
        rec.update({"alg_bytes": nb, "hbm_frac": nb / (rec["us_per_call"] * 1e-6) / 1e9 / hbm,
                    "speedup_vs_plain_decode": dec_us / rec["us_per_call"]})
    flops_pass = 2.0 * wl.num_q_heads * wl.window * sum(lens) * wl.head_dim
    seg_tokens = sum((T // wl.segment_len) * wl.segment_len for T in lens)
    kv_seg_bytes = seg_tokens * wl.num_kv_heads * wl.head_dim * 2
    chan_tokens = seg_tokens * wl.num_kv_heads
    work = {
        "score_pass1": ("tensor", flops_pass, sum(lens) * wl.num_kv_heads),
        "score_pass2": ("tensor", 2.0 * wl.num_q_heads * wl.window * seg_tokens * wl.head_dim,
                        chan_tokens),
        # K rows in; a 16-byte keep mask and the fp64 g_t out per token
        "chan_topc": ("hbm", kv_seg_bytes + chan_tokens * (16 + 8), chan_tokens),
        "pack": ("hbm", 2 * used, chan_tokens),   # gathers about as many bytes as it writes
        "decode": ("hbm", dec_bytes, None),
    }
    kernels = {}
    tot_prof = sum(t for t, _ in prof.values())
    for name, (tot, n) in prof.items():
        if n:
            kernels[name] = {"launches": n, "avg_us": 1e3 * tot / n, "share": tot / max(tot_prof, 1e-12)}
    dominant = max(kernels, key=lambda k_: kernels[k_]["avg_us"] * kernels[k_]["launches"])
    kind, amount, toks = work.get(dominant, ("hbm", 0.0, None))
    avg_s = kernels[dominant]["avg_us"] * 1e-6
    traffic, traffic_note = profiled_traffic(dominant, toks) if toks else (None, "not captured")
    roof = roofline_of(kind, amount, avg_s, hbm, tf_burst, tf_sust, src)
    roof.update({"traffic": traffic, "kernel": dominant})
    roof["algorithmic_per_launch"] = amount
    roof["traffic_source"] = traffic_note
    gpu_launches = sum(v_["launches"] for v_ in kernels.values())
    # the scoring contraction, both passes (executed MMA flops = algorithmic)
    scoring = None
    if "score_pass1" in kernels and "score_pass2" in kernels:
        scoring = scoring_of(flops_pass, work["score_pass2"][1], kernels["score_pass1"]["avg_us"],
                             kernels["score_pass2"]["avg_us"], tf_burst, tf_sust, src)
    comp_alg = compress_alg_bytes(wl, lens, used)

    # ---- end to end through the public API with host buffers
    e2e = None
    if not args.no_e2e:
        hk, hv, hqw, hq = (t.cpu().pin_memory() for t in (k, v, qw, q))
        hkn, hvn = kn.cpu().pin_memory(), vn.cpu().pin_memory()
        hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = sum(t.numel() * t.element_size() for t in (hk, hv, hqw, hq, hkn, hvn))
        if bt is not None:
            hbt = bt.cpu().pin_memory()
            h2d += hbt.numel() * 4
        d2h = hout.numel() * hout.element_size()
        evs = []
        for i in range(max(3, args.warmup) + args.steps):
            a, b_ = event_pair(torch)
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
        del hk, hv, hqw, hq

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        units = cpu_sample_units(wl, args.seed, cpu_sample_size())
        xs = host_units(bat, wl, units)
        wall, phases, nb = oracle_sample(wl, xs, scale)
        cpu = cpu_record(wl, units, xs, wall, phases, nb)
        del xs

    extras = None
    if world == 1 and not args.no_extras:
        del bat, k, v, qw, q, cc, ws_c, dv
        torch.cuda.empty_cache()
        extras = {}
        for name in EXTRA_WORKLOADS:
            if name != wl.name:
                extras[name] = measure_extra(name, B, synth, torch, dev, stream, flush, hbm,
                                             max(args.steps, 5))

    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return
    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f16", "data": "synthetic",
        "config": config_of(wl, lens, world),
        "decode": {"us_per_step": dec_us, "bytes_per_step": dec_bytes,
                   "hbm_gbs": dec_bytes / (dec_us * 1e-6) / 1e9,
                   "hbm_frac": dec_bytes / (dec_us * 1e-6) / 1e9 / hbm,
                   "hbm_frac_of_8tbs_nominal": dec_bytes / (dec_us * 1e-6) / 1e9 / 8000.0,
                   "graph_us_per_call": graph_us,
                   "graph_note": "100 back-to-back calls in one CUDA graph, no flush between them",
                   "budget1_us": dense_dec_us,
                   "speedup_vs_budget1": (dense_dec_us / dec_us) if dense_dec_us else None},
        "decode_select": {"rates": sel_rec,
                          "note": "decode-time token selection: candidate scores, top-n per unit, "
                                  "attention over the kept tokens and the dense tail; L2 flushed"},
        "compress": {"us": comp_us, "gbs": nbytes / (comp_us * 1e-6) / 1e9,
                     "alg_bytes": comp_alg, "hbm_frac": comp_alg / (comp_us * 1e-6) / 1e9 / hbm},
        "scoring": scoring,
        "extras": extras,
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
