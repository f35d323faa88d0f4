"""ctypes front end of the fp64 CPU oracle (kv2d_oracle.c).

TEST INFRASTRUCTURE ONLY: the test suite, the package smoke check and the
benchmark's CPU-baseline leg are the only callers.  The product library never
imports this module and this module never imports the product package.

Every function below hands numpy arrays to the C oracle; the arithmetic lives
in kv2d_oracle.c, whose header cites the passages each step follows.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kv2d_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

FULL, TOK, CH, BOTH = 0, 1, 2, 3
OK, INFEASIBLE = 0, 2


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (fp64, no fused multiply-add)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".{os.getpid()}.tmp"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
             "-shared", _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


class Params(C.Structure):
    _fields_ = [("d", C.c_int32), ("G", C.c_int32), ("S", C.c_int32), ("W", C.c_int32),
                ("r", C.c_int32), ("c", C.c_int32), ("beta", C.c_double), ("scale", C.c_double),
                ("chunk_len", C.c_int32), ("chunk_budget", C.c_int32)]


_lib = None
_lock = threading.Lock()


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = C.CDLL(build())
            P = C.POINTER
            dp, u8p, i32p, i64p, u16p = (P(C.c_double), P(C.c_uint8), P(C.c_int32),
                                         P(C.c_int64), P(C.c_uint16))
            pp = P(Params)
            L.orc_half_to_double.argtypes = [C.c_uint16]
            L.orc_half_to_double.restype = C.c_double
            L.orc_win_stats.argtypes = [pp, dp, dp]
            L.orc_score.argtypes = [pp, C.c_int, C.c_int, dp, dp, dp, dp]
            L.orc_score.restype = C.c_int
            L.orc_channel.argtypes = [pp, C.c_int, dp, dp, u8p, dp]
            L.orc_topr.argtypes = [pp, dp, u8p]
            L.orc_topr_chunks.argtypes = [pp, dp, u8p]
            L.orc_segment_errors.argtypes = [pp, dp, dp, u8p, dp]
            L.orc_segment_bytes.argtypes = [pp, C.c_int]
            L.orc_segment_bytes.restype = C.c_int64
            L.orc_hull.argtypes = [pp, dp, i32p, dp, i64p]
            L.orc_hull.restype = C.c_int
            L.orc_budget_bytes.argtypes = [pp, C.c_int]
            L.orc_budget_bytes.restype = C.c_int64
            L.orc_budget.argtypes = [pp, C.c_int, i32p, i32p, dp, i64p, i32p, i64p]
            L.orc_budget.restype = C.c_int
            L.orc_pack_segment.argtypes = [pp, C.c_int, u16p, u16p, u8p, u8p, u8p]
            L.orc_pack_segment.restype = C.c_int64
            L.orc_compress_unit.argtypes = [pp, C.c_int, C.c_int, u16p, u16p, dp, dp, dp, dp,
                                            dp, dp, dp, dp, u8p, u8p, dp, i32p, i64p, u8p,
                                            C.c_int64, i64p]
            L.orc_compress_unit.restype = C.c_int
            L.orc_decode.argtypes = [pp, C.c_int, u8p, i64p, i32p, C.c_int, dp, dp, dp, dp]
            L.orc_select_scores.argtypes = [pp, C.c_int, u8p, i64p, i32p, dp, dp]
            L.orc_select_scores.restype = C.c_int64
            L.orc_select_count.argtypes = [pp, C.c_int, C.c_int64, C.c_double]
            L.orc_select_count.restype = C.c_int64
            L.orc_select_tokens.argtypes = [C.c_int64, dp, C.c_int64, u8p]
            L.orc_decode_select.argtypes = [pp, C.c_int, u8p, i64p, i32p, u8p, C.c_int, dp, dp,
                                            dp, dp]
            _lib = L
    return _lib


def params(d, G, S, W, r, c, beta, scale=None, chunk_len=0, chunk_budget=0) -> Params:
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    return Params(int(d), int(G), int(S), int(W), int(r), int(c), float(beta), float(scale),
                  int(chunk_len), int(chunk_budget))


def _p(a, ct):
    return a.ctypes.data_as(C.POINTER(ct))


def _f64(x):
    return np.ascontiguousarray(x, dtype=np.float64)


def _u16(x):
    x = np.ascontiguousarray(x)
    if x.dtype == np.float16:
        x = x.view(np.uint16)
    return np.ascontiguousarray(x, dtype=np.uint16)


def half_to_double(bits: int) -> float:
    return lib().orc_half_to_double(int(bits))


def win_stats(p: Params, qw) -> np.ndarray:
    qw = _f64(qw)
    a = np.zeros(p.d)
    lib().orc_win_stats(C.byref(p), _p(qw, C.c_double), _p(a, C.c_double))
    return a


def score(p: Params, T: int, r0: int, K, qw):
    """K: region keys [T-r0][d]; qw: [G*W][d].  Returns (lse[G*W], s[T-r0])."""
    K, qw = _f64(K), _f64(qw)
    lse = np.zeros(p.G * p.W)
    s = np.zeros(T - r0)
    rc = lib().orc_score(C.byref(p), T, r0, _p(K, C.c_double), _p(qw, C.c_double),
                         _p(lse, C.c_double), _p(s, C.c_double))
    if rc != 0:
        raise ValueError("window larger than the region")
    return lse, s


def channel(p: Params, K, a):
    K, a = _f64(K), _f64(a)
    n = K.shape[0]
    cidx = np.zeros((n, p.c), np.uint8)
    g = np.zeros(n)
    lib().orc_channel(C.byref(p), n, _p(K, C.c_double), _p(a, C.c_double),
                      _p(cidx, C.c_uint8), _p(g, C.c_double))
    return cidx, g


def topr(p: Params, s_seg) -> np.ndarray:
    s_seg = _f64(s_seg)
    t = np.zeros(p.r, np.uint8)
    lib().orc_topr(C.byref(p), _p(s_seg, C.c_double), _p(t, C.c_uint8))
    return t


def topr_chunks(p: Params, s_seg) -> np.ndarray:
    """The Token2Chunk variant of the kept tokens of one segment."""
    s_seg = _f64(s_seg)
    t = np.zeros(p.r, np.uint8)
    lib().orc_topr_chunks(C.byref(p), _p(s_seg, C.c_double), _p(t, C.c_uint8))
    return t


def segment_errors(p: Params, s_seg, g_seg, tidx) -> np.ndarray:
    s_seg, g_seg = _f64(s_seg), _f64(g_seg)
    tidx = np.ascontiguousarray(tidx, np.uint8)
    E = np.zeros(4)
    lib().orc_segment_errors(C.byref(p), _p(s_seg, C.c_double), _p(g_seg, C.c_double),
                             _p(tidx, C.c_uint8), _p(E, C.c_double))
    return E


def segment_bytes(p: Params, strategy: int) -> int:
    return int(lib().orc_segment_bytes(C.byref(p), int(strategy)))


def hull(p: Params, E):
    E = _f64(E)
    verts = np.zeros(4, np.int32)
    eff = np.zeros(3)
    db = np.zeros(3, np.int64)
    nv = lib().orc_hull(C.byref(p), _p(E, C.c_double), _p(verts, C.c_int32),
                        _p(eff, C.c_double), _p(db, C.c_int64))
    return verts[:nv].copy(), eff[:nv - 1].copy(), db[:nv - 1].copy()


def budget_bytes(p: Params, nseg: int) -> int:
    return int(lib().orc_budget_bytes(C.byref(p), int(nseg)))


def budget(p: Params, E_all):
    """E_all: [nseg][4].  Returns (status, strategies[nseg], used_bytes)."""
    E_all = _f64(E_all).reshape(-1, 4)
    nseg = E_all.shape[0]
    nv = np.zeros(max(nseg, 1), np.int32)
    verts = np.zeros((max(nseg, 1), 4), np.int32)
    eff = np.zeros((max(nseg, 1), 3))
    db = np.zeros((max(nseg, 1), 3), np.int64)
    for j in range(nseg):
        nv[j] = lib().orc_hull(C.byref(p), _p(np.ascontiguousarray(E_all[j]), C.c_double),
                               _p(verts[j], C.c_int32), _p(eff[j], C.c_double),
                               _p(db[j], C.c_int64))
    strat = np.zeros(max(nseg, 1), np.int32)
    used = np.zeros(1, np.int64)
    st = lib().orc_budget(C.byref(p), nseg, _p(nv, C.c_int32), _p(verts, C.c_int32),
                          _p(eff, C.c_double), _p(db, C.c_int64), _p(strat, C.c_int32),
                          _p(used, C.c_int64))
    return st, strat[:nseg].copy(), int(used[0])


def pack_segment(p: Params, strategy, K16, V16, tidx, cidx_all) -> np.ndarray:
    K16, V16 = _u16(K16), _u16(V16)
    tidx = np.ascontiguousarray(tidx, np.uint8)
    cidx_all = np.ascontiguousarray(cidx_all, np.uint8)
    out = np.zeros(segment_bytes(p, strategy), np.uint8)
    n = lib().orc_pack_segment(C.byref(p), int(strategy), _p(K16, C.c_uint16),
                               _p(V16, C.c_uint16), _p(tidx, C.c_uint8),
                               _p(cidx_all, C.c_uint8), _p(out, C.c_uint8))
    assert n == out.size
    return out


def compress_unit(p: Params, T: int, r0: int, K16, V16, qw16, a_in=None, s_in=None,
                  arena_base: int = 0):
    """One (sequence, KV head) unit.  K16/V16: region rows [T-r0][d] fp16;
    qw16: window rows [G*W][d] fp16.  a_in/s_in: optional fed values."""
    K16, V16 = _u16(K16), _u16(V16)
    Kd = K16.view(np.float16).astype(np.float64)
    qw = _u16(qw16).view(np.float16).astype(np.float64)
    n = T - r0
    nseg = n // p.S
    a = np.zeros(p.d)
    lse = np.zeros(p.G * p.W)
    s = np.zeros(n)
    g = np.zeros(max(nseg * p.S, 1))
    cidx = np.zeros((max(nseg * p.S, 1), p.c), np.uint8)
    tidx = np.zeros((max(nseg, 1), p.r), np.uint8)
    E = np.zeros((max(nseg, 1), 4))
    strat = np.zeros(max(nseg, 1), np.int32)
    offs = np.zeros(max(nseg, 1), np.int64)
    cap = arena_base + nseg * segment_bytes(p, FULL) + 16
    arena = np.zeros(cap, np.uint8)
    used = np.zeros(1, np.int64)
    a_keep = _f64(a_in) if a_in is not None else None
    s_keep = _f64(s_in) if s_in is not None else None
    a_ptr = _p(a_keep, C.c_double) if a_keep is not None else None
    s_ptr = _p(s_keep, C.c_double) if s_keep is not None else None
    st = lib().orc_compress_unit(
        C.byref(p), T, r0, _p(K16, C.c_uint16), _p(V16, C.c_uint16), _p(Kd, C.c_double),
        _p(qw, C.c_double), a_ptr, s_ptr, _p(a, C.c_double), _p(lse, C.c_double),
        _p(s, C.c_double), _p(g, C.c_double), _p(cidx, C.c_uint8), _p(tidx, C.c_uint8),
        _p(E, C.c_double), _p(strat, C.c_int32), _p(offs, C.c_int64), _p(arena, C.c_uint8),
        arena_base, _p(used, C.c_int64))
    if st < 0:
        raise ValueError("bad arguments to compress_unit")
    return dict(status=st, a=a, lse=lse, s=s, g=g[:nseg * p.S], cidx=cidx[:nseg * p.S],
                tidx=tidx[:nseg], E=E[:nseg], strat=strat[:nseg], offs=offs[:nseg],
                used=int(used[0]), arena=arena[:arena_base + int(used[0])], nseg=nseg)


def decode_unit(p: Params, arena, offs, strat, Kt16, Vt16, q16) -> np.ndarray:
    """Attention of the unit's G heads (q16 [G][d]) over the packed segments
    (arena bytes, offs, strat) and dense tail rows Kt16/Vt16 [n][d]."""
    arena = np.ascontiguousarray(arena, np.uint8)
    if arena.size == 0:
        arena = np.zeros(16, np.uint8)
    offs = np.ascontiguousarray(offs, np.int64)
    strat = np.ascontiguousarray(strat, np.int32)
    nseg = strat.size
    Kt = _u16(Kt16).view(np.float16).astype(np.float64).reshape(-1, p.d)
    Vt = _u16(Vt16).view(np.float16).astype(np.float64).reshape(-1, p.d)
    if Kt.shape[0] == 0:
        Kt = np.zeros((1, p.d))
        Vt = np.zeros((1, p.d))
        n_tail = 0
    else:
        n_tail = Kt.shape[0]
    q = _u16(q16).view(np.float16).astype(np.float64).reshape(p.G, p.d)
    q = np.ascontiguousarray(q)
    out = np.zeros((p.G, p.d))
    offs_ = offs if offs.size else np.zeros(1, np.int64)
    strat_ = strat if strat.size else np.zeros(1, np.int32)
    lib().orc_decode(C.byref(p), nseg, _p(arena, C.c_uint8), _p(offs_, C.c_int64),
                     _p(strat_, C.c_int32), n_tail, _p(np.ascontiguousarray(Kt), C.c_double),
                     _p(np.ascontiguousarray(Vt), C.c_double), _p(q, C.c_double),
                     _p(out, C.c_double))
    return out


def _seg_args(arena, offs, strat):
    arena = np.ascontiguousarray(arena, np.uint8)
    if arena.size == 0:
        arena = np.zeros(16, np.uint8)
    offs = np.ascontiguousarray(offs, np.int64)
    strat = np.ascontiguousarray(strat, np.int32)
    nseg = strat.size
    offs_ = offs if offs.size else np.zeros(1, np.int64)
    strat_ = strat if strat.size else np.zeros(1, np.int32)
    return arena, offs_, strat_, nseg


def select_scores(p: Params, arena, offs, strat, q16):
    """Decode-time selection scores of every candidate slot j*S + i: the
    largest logit over the G heads (-inf past a segment's kept tokens).
    Returns (score[nseg*S], number of candidates)."""
    arena, offs_, strat_, nseg = _seg_args(arena, offs, strat)
    q = np.ascontiguousarray(_u16(q16).view(np.float16).astype(np.float64).reshape(p.G, p.d))
    score = np.zeros(max(nseg * p.S, 1))
    n = lib().orc_select_scores(C.byref(p), nseg, _p(arena, C.c_uint8), _p(offs_, C.c_int64),
                                _p(strat_, C.c_int32), _p(q, C.c_double), _p(score, C.c_double))
    return score[:nseg * p.S], int(n)


def select_count(p: Params, nseg: int, ncand: int, rho: float) -> int:
    return int(lib().orc_select_count(C.byref(p), int(nseg), int(ncand), float(rho)))


def select_tokens(score, n_sel: int) -> np.ndarray:
    """Flags of the n_sel largest finite scores, ties to the lower slot."""
    score = _f64(score)
    sel = np.zeros(max(score.size, 1), np.uint8)
    lib().orc_select_tokens(score.size, _p(score if score.size else np.zeros(1), C.c_double),
                            int(n_sel), _p(sel, C.c_uint8))
    return sel[:score.size]


def decode_select(p: Params, arena, offs, strat, sel, Kt16, Vt16, q16) -> np.ndarray:
    """Attention of the G heads over the selected candidates (flags per slot
    j*S + i) and the dense tail rows."""
    arena, offs_, strat_, nseg = _seg_args(arena, offs, strat)
    sel = np.ascontiguousarray(sel, np.uint8)
    sel_ = sel if sel.size else np.zeros(1, np.uint8)
    Kt = _u16(Kt16).view(np.float16).astype(np.float64).reshape(-1, p.d)
    Vt = _u16(Vt16).view(np.float16).astype(np.float64).reshape(-1, p.d)
    n_tail = Kt.shape[0]
    if n_tail == 0:
        Kt = np.zeros((1, p.d))
        Vt = np.zeros((1, p.d))
    q = np.ascontiguousarray(_u16(q16).view(np.float16).astype(np.float64).reshape(p.G, p.d))
    out = np.zeros((p.G, p.d))
    lib().orc_decode_select(C.byref(p), nseg, _p(arena, C.c_uint8), _p(offs_, C.c_int64),
                            _p(strat_, C.c_int32), _p(sel_, C.c_uint8), n_tail,
                            _p(np.ascontiguousarray(Kt), C.c_double),
                            _p(np.ascontiguousarray(Vt), C.c_double), _p(q, C.c_double),
                            _p(out, C.c_double))
    return out


def parallel_map(fn, items, threads=None):
    """Runs fn over independent units on host threads (ctypes releases the
    GIL inside the C oracle, so the units run concurrently)."""
    threads = threads or os.cpu_count() or 1
    with ThreadPoolExecutor(max_workers=threads) as ex:
        return list(ex.map(fn, items))
