"""Runs the CUDA path through the C ABI and compares it with the CPU oracle.

Comparison protocol (per unit = (sequence, KV head)):
  1. a_d, lse, s_t against the oracle's fp64 values (relative 1e-4; s has an
     absolute floor of 1e-6 * max s because tiny masses have no meaningful
     relative error);
  2. the oracle is then fed the GPU's fp32 a_d and s_t: g_t, the error
     proxies, strategies, descriptors, used bytes and every arena byte must
     match exactly (integer / byte work is bit-exact);
  3. decode output (fp16) against the oracle's fp64 decode on the same arena:
     max abs error <= 2e-3.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
import torch

from kv_cache_compression_kv2d_b200 import binding as B
from kv_cache_compression_kv2d_b200 import synth

TOL_REL = 1e-4
TOL_OUT = 2e-3


@dataclass
class GpuCase:
    wl: synth.Workload
    batch: synth.Batch
    p: B.kv2d_params
    cc: B.CompressedCache
    dv: B.kv2d_dense
    seq_len: torch.Tensor       # device int32
    comp_end_host: list
    dbg: dict
    ws: torch.Tensor


def params_for(wl: synth.Workload, budget=None, keep_channels=None, keep_tokens=None,
               chunk_len=0, chunk_budget=0):
    scale = float(np.float32(1.0 / math.sqrt(wl.head_dim)))
    return B.params(wl.head_dim, wl.num_q_heads, wl.num_kv_heads, wl.segment_len, wl.window,
                    keep_tokens or wl.r, keep_channels or wl.c,
                    wl.budget if budget is None else budget, scale, chunk_len, chunk_budget)


def oracle_params(orc, p: B.kv2d_params):
    return orc.params(p.head_dim, p.num_q_heads // p.num_kv_heads, p.segment_len, p.window,
                      p.keep_tokens, p.keep_channels, float(np.float32(p.budget)),
                      float(np.float32(p.scale)), p.chunk_len, p.chunk_budget if p.chunk_len else 0)


def to_device(batch: synth.Batch, device="cuda") -> synth.Batch:
    bt = batch.block_table.to(device) if batch.block_table is not None else None
    return synth.Batch(batch.wl, batch.seq_len, batch.k.to(device), batch.v.to(device),
                       batch.qw.to(device), batch.q.to(device), batch.capacity, bt,
                       batch.mu.to(device) if batch.mu is not None else None)


def make_run(wl, batch_dev, p, max_tokens=None):
    B_ = wl.batch
    max_tokens = max_tokens or batch_dev.capacity
    cc = B.CompressedCache(p, B_, max_tokens)
    if batch_dev.block_table is not None:
        dv = B.dense(batch_dev.k, batch_dev.v, batch_dev.block_table, wl.block_size)
    else:
        dv = B.dense(batch_dev.k, batch_dev.v)
    seq = batch_dev.seq_len.to(torch.int32).cuda()
    ws = B.workspace(B.kv2d_workspace_bytes(p, B.OP_COMPRESS, B_, max_tokens))
    return GpuCase(wl, batch_dev, p, cc, dv, seq, [0] * B_, {}, ws)


def compress(run: GpuCase, seq_host=None, expect_bits=0):
    wl, p = run.wl, run.p
    Bn = wl.batch
    seq_host = [int(x) for x in (seq_host if seq_host is not None else run.seq_len.cpu().tolist())]
    regions = [seq_host[b] - run.comp_end_host[b] for b in range(Bn)]
    rmax = max(max(regions), 1)
    nseg_max = max(max(regions) // wl.segment_len, 1)
    units = Bn * wl.num_kv_heads
    dbg = dict(a=torch.full((units, wl.head_dim), float("nan"), device="cuda"),
               lse=torch.full((Bn, wl.num_q_heads, wl.window), float("nan"), device="cuda"),
               s=torch.full((units, rmax), float("nan"), device="cuda"),
               g=torch.full((units, rmax), float("nan"), dtype=torch.float64, device="cuda"),
               E=torch.full((units, nseg_max, 4), float("nan"), dtype=torch.float64,
                            device="cuda"))
    need = B.kv2d_workspace_bytes(p, B.OP_COMPRESS, Bn, rmax)
    if run.ws.numel() < need:
        run.ws = B.workspace(need)
    d = B.kv2d_debug(dbg["a"].data_ptr(), dbg["lse"].data_ptr(), dbg["s"].data_ptr(),
                     dbg["g"].data_ptr(), dbg["E"].data_ptr(), rmax, nseg_max)
    ce_before = list(run.comp_end_host)
    B.kv2d_compress(p, Bn, seq_host, ce_before, run.dv, run.batch.qw, run.cc.struct, run.ws, d)
    torch.cuda.synchronize()
    bits = B.kv2d_read_status(run.ws)
    assert bits == expect_bits, f"device status bits {bits:#x}, expected {expect_bits:#x}"
    run.dbg = dict(dbg, ce_before=ce_before, seq_host=seq_host)
    run.comp_end_host = [ce_before[b] + (regions[b] // wl.segment_len) * wl.segment_len
                         for b in range(Bn)]
    return run


def unit_inputs(run: GpuCase, b: int, h: int, t0: int, t1: int):
    k, v = synth.dense_rows(run.batch, b, h, t0, t1)
    return k.cpu().numpy(), v.cpu().numpy()


def unit_qw(run: GpuCase, b: int, h: int):
    G, W, d = run.wl.group, run.wl.window, run.wl.head_dim
    return run.batch.qw[b, h * G:(h + 1) * G].reshape(G * W, d).cpu().numpy()


def oracle_scores(orc, run: GpuCase, b: int, h: int, threads=None):
    """The oracle's own a_d, lse and s_t of unit (b, h) for the latest
    compress() call, scored one query head at a time on host threads: head
    g's W window rows are an independent single-head problem over the same
    keys (its rows' lse values are those of the full call, and s_t is the
    sum over heads of each head's share).  Returns (a, lse[G*W], s[n])."""
    wl, p = run.wl, run.p
    po = oracle_params(orc, p)
    T = run.dbg["seq_host"][b]
    r0 = run.dbg["ce_before"][b]
    G, W, d = wl.group, wl.window, wl.head_dim
    K16, _ = unit_inputs(run, b, h, r0, T)
    Kd = K16.astype(np.float64)
    qw = unit_qw(run, b, h).astype(np.float64)
    po1 = orc.params(d, 1, p.segment_len, W, p.keep_tokens, p.keep_channels,
                     float(np.float32(p.budget)), float(np.float32(p.scale)))
    parts = orc.parallel_map(lambda g: orc.score(po1, T, r0, Kd, qw[g * W:(g + 1) * W]),
                             list(range(G)), threads=threads)
    lse = np.concatenate([lp for lp, _ in parts])
    s = np.zeros(T - r0)
    for _, sp in parts:
        s += sp
    return orc.win_stats(po, qw), lse, s


def check_scores(run: GpuCase, b: int, h: int, scores):
    """a_d, lse and s_t of unit (b, h) against the oracle's (a, lse, s)."""
    wl = run.wl
    a_ref, lse_ref, s_ref = scores
    u = b * wl.num_kv_heads + h
    n = run.dbg["seq_host"][b] - run.dbg["ce_before"][b]
    nS = (n // wl.segment_len) * wl.segment_len
    a_gpu = run.dbg["a"][u].double().cpu().numpy()
    s_gpu = run.dbg["s"][u, :nS].double().cpu().numpy()
    lse_gpu = run.dbg["lse"][b, h * wl.group:(h + 1) * wl.group].reshape(-1).double().cpu().numpy()
    assert np.max(np.abs(a_gpu - a_ref) / np.maximum(np.abs(a_ref), 1e-30)) < 1e-5
    assert np.max(np.abs(lse_gpu - lse_ref) / np.maximum(1.0, np.abs(lse_ref))) < TOL_REL, \
        f"lse mismatch {np.max(np.abs(lse_gpu - lse_ref))}"
    s_seg = s_ref[:nS]
    floor = 1e-6 * np.max(s_seg)
    err = np.abs(s_gpu - s_seg) / np.maximum(np.abs(s_seg), floor)
    assert np.max(err) < TOL_REL, f"s mismatch {np.max(err)} at {np.argmax(err)}"
    return float(np.max(err))


def end_to_end_unit(orc, run: GpuCase, b: int, h: int, scores, q: torch.Tensor):
    """The fully independent end-to-end oracle for unit (b, h): the oracle's
    own a_d and s_t (scores), its own selection and packing of the region of
    the latest compress() call, and its decode of q over that arena plus the
    unit's dense tail.  Returns (strategy agreement with the GPU as
    (agreeing, total), max abs difference between the GPU's decode output
    (out, fp16 [B][Hq][d] on the host) and the oracle's)."""
    wl, p = run.wl, run.p
    po = oracle_params(orc, p)
    a_ref, _, s_ref = scores
    T = run.dbg["seq_host"][b]
    r0 = run.dbg["ce_before"][b]
    S = wl.segment_len
    u = b * wl.num_kv_heads + h
    K16, V16 = unit_inputs(run, b, h, r0, T)
    ref = orc.compress_unit(po, T, r0, K16, V16, unit_qw(run, b, h), a_in=a_ref, s_in=s_ref)
    assert ref["status"] == 0
    nseg = ref["nseg"]
    desc = run.cc.desc[u].cpu().numpy().view(np.uint64)
    seg0 = r0 // S
    strat_gpu = ((desc[seg0:seg0 + nseg] >> np.uint64(32)) & np.uint64(255)).astype(np.int32)
    agree = int(np.sum(strat_gpu == ref["strat"]))
    # decode of q over the oracle's own arena (segments of this call) and the
    # dense tail after them; only units compressed in one call are compared
    assert r0 == 0, "end-to-end decode compares units compressed in one call"
    Tn = int(run.seq_len[b])
    ce = nseg * S
    Kt, Vt = unit_inputs(run, b, h, ce, Tn)
    G = wl.group
    o_ref = orc.decode_unit(po, ref["arena"], ref["offs"], ref["strat"], Kt, Vt,
                            q[b, h * G:(h + 1) * G].cpu().numpy())
    return (agree, nseg), o_ref


def check_compress_unit(orc, run: GpuCase, b: int, h: int, independent: bool = True,
                        arena_before=None, scores=None):
    """Parity of one unit after the latest compress() call.  With scores
    (the oracle's (a, lse, s), e.g. from oracle_scores) those are compared
    instead of scoring the unit again."""
    wl, p = run.wl, run.p
    po = oracle_params(orc, p)
    u = b * wl.num_kv_heads + h
    T = run.dbg["seq_host"][b]
    r0 = run.dbg["ce_before"][b]
    n = T - r0
    S = wl.segment_len
    nseg = n // S
    if nseg == 0:
        return None
    K16, V16 = unit_inputs(run, b, h, r0, T)
    qw16 = unit_qw(run, b, h)
    a_gpu = run.dbg["a"][u].double().cpu().numpy()
    s_gpu = run.dbg["s"][u, :n].double().cpu().numpy()
    g_gpu = run.dbg["g"][u, :nseg * S].cpu().numpy()
    E_gpu = run.dbg["E"][u, :nseg].cpu().numpy()
    lse_gpu = run.dbg["lse"][b, h * wl.group:(h + 1) * wl.group].reshape(-1).double().cpu().numpy()

    if scores is not None:
        check_scores(run, b, h, scores)
    elif independent:
        a_ref = orc.win_stats(po, qw16.astype(np.float64))
        assert np.max(np.abs(a_gpu - a_ref) / np.maximum(np.abs(a_ref), 1e-30)) < 1e-5
        lse_ref, s_ref = orc.score(po, T, r0, K16.astype(np.float64), qw16.astype(np.float64))
        assert np.max(np.abs(lse_gpu - lse_ref) / np.maximum(1.0, np.abs(lse_ref))) < TOL_REL, \
            f"lse mismatch {np.max(np.abs(lse_gpu - lse_ref))}"
        s_seg = s_ref[:nseg * S]
        floor = 1e-6 * np.max(s_seg)
        err = np.abs(s_gpu[:nseg * S] - s_seg) / np.maximum(np.abs(s_seg), floor)
        assert np.max(err) < TOL_REL, f"s mismatch {np.max(err)} at {np.argmax(err)}"

    # fed mode: the oracle's selection on the GPU's fp32 scores
    s_fed = np.zeros(n)
    s_fed[:nseg * S] = s_gpu[:nseg * S]
    ref = orc.compress_unit(po, T, r0, K16, V16, qw16, a_in=a_gpu, s_in=s_fed,
                            arena_base=0)
    assert ref["status"] == 0
    assert np.array_equal(g_gpu, ref["g"]), "g_t differs bitwise"
    assert np.array_equal(E_gpu, ref["E"]), "error proxies differ bitwise"
    desc = run.cc.desc[u].cpu().numpy().view(np.uint64)
    used = int(run.cc.used_bytes[u])
    seg0 = r0 // S
    strat_gpu = ((desc[seg0:seg0 + nseg] >> np.uint64(32)) & np.uint64(255)).astype(np.int32)
    offs_gpu = (desc[seg0:seg0 + nseg] & np.uint64(0xffffffff)).astype(np.int64) * 16
    assert np.array_equal(strat_gpu, ref["strat"]), "strategies differ"
    base = int(offs_gpu[0])
    assert np.array_equal(offs_gpu - base, ref["offs"]), "offsets differ"
    assert used - base == ref["used"], "used bytes differ"
    assert int(run.cc.n_segs[u]) == seg0 + nseg
    assert int(run.cc.comp_end[b]) == r0 + nseg * S
    arena = run.cc.arena[u * run.cc.arena_stride: u * run.cc.arena_stride + used].cpu().numpy()
    assert np.array_equal(arena[base:used], ref["arena"][:ref["used"]]), "arena bytes differ"
    return dict(strat=ref["strat"], nseg=nseg)


def gpu_decode(run: GpuCase, q: torch.Tensor, cc: B.CompressedCache | None = None,
               max_seq=None, expect_bits=0):
    wl, p = run.wl, run.p
    cc = cc or run.cc
    out = torch.full((wl.batch, wl.num_q_heads, wl.head_dim), float("nan"),
                     dtype=torch.float16, device="cuda")
    ms = max_seq or run.batch.capacity
    ws = B.workspace(B.kv2d_workspace_bytes(p, B.OP_DECODE, wl.batch, ms))
    B.kv2d_decode_attn(p, wl.batch, cc.struct, run.dv, run.seq_len, ms, q, out, ws)
    torch.cuda.synchronize()
    bits = B.kv2d_read_status(ws)
    if expect_bits is not None:
        assert bits == expect_bits, f"device status bits {bits:#x}, expected {expect_bits:#x}"
    return out


def oracle_decode_unit(orc, run: GpuCase, b: int, h: int, q: torch.Tensor,
                       cc: B.CompressedCache | None = None):
    """Oracle decode of unit (b, h) over the arena and descriptors the cache
    holds (bytes already proven equal to the oracle's own packing)."""
    wl, p = run.wl, run.p
    po = oracle_params(orc, p)
    cc = cc or run.cc
    u = b * wl.num_kv_heads + h
    nsg = int(cc.n_segs[u])
    used = int(cc.used_bytes[u])
    ce = int(cc.comp_end[b])
    T = int(run.seq_len[b])
    desc = cc.desc[u, :nsg].cpu().numpy().view(np.uint64)
    strat = ((desc >> np.uint64(32)) & np.uint64(255)).astype(np.int32)
    offs = (desc & np.uint64(0xffffffff)).astype(np.int64) * 16
    arena = cc.arena[u * cc.arena_stride: u * cc.arena_stride + used].cpu().numpy()
    Kt, Vt = unit_inputs(run, b, h, ce, T)
    G = wl.group
    qh = q[b, h * G:(h + 1) * G].cpu().numpy()
    return orc.decode_unit(po, arena, offs, strat, Kt, Vt, qh)


def unit_cache(run: GpuCase, b: int, h: int, cc: B.CompressedCache | None = None):
    """The packed bytes, offsets and strategies of unit (b, h) and the dense
    tail rows after its segments."""
    cc = cc or run.cc
    u = b * run.wl.num_kv_heads + h
    nsg = int(cc.n_segs[u])
    used = int(cc.used_bytes[u])
    ce = int(cc.comp_end[b])
    T = int(run.seq_len[b])
    desc = cc.desc[u, :nsg].cpu().numpy().view(np.uint64)
    strat = ((desc >> np.uint64(32)) & np.uint64(255)).astype(np.int32)
    offs = (desc & np.uint64(0xffffffff)).astype(np.int64) * 16
    arena = cc.arena[u * cc.arena_stride: u * cc.arena_stride + used].cpu().numpy()
    Kt, Vt = unit_inputs(run, b, h, ce, T)
    return arena, offs, strat, Kt, Vt


def gpu_decode_select(run: GpuCase, q: torch.Tensor, rate: float, max_seq=None):
    """kv2d_decode_attn_select with its per-slot scores and kept flags."""
    wl, p = run.wl, run.p
    ms = max_seq or run.batch.capacity
    units = wl.batch * wl.num_kv_heads
    slots = -(-(ms // wl.segment_len * wl.segment_len) // 4) * 4
    slots = max(slots, 4)
    out = torch.full((wl.batch, wl.num_q_heads, wl.head_dim), float("nan"), dtype=torch.float16,
                     device="cuda")
    score = torch.full((units, slots), float("nan"), device="cuda")
    sel = torch.full((units, slots), 7, dtype=torch.uint8, device="cuda")
    ws = B.workspace(B.kv2d_workspace_bytes(p, B.OP_DECODE_SELECT, wl.batch, ms))
    B.kv2d_decode_attn_select(p, wl.batch, run.cc.struct, run.dv, run.seq_len, ms, q, out, rate, ws,
                              score, sel)
    torch.cuda.synchronize()
    bits = B.kv2d_read_status(ws)
    assert bits == 0, f"device status bits {bits:#x}"
    return out, score, sel
