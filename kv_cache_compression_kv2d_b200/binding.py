"""ctypes binding of the kv2d C ABI (include/kv2d.h).

Argument marshalling only: every step of compression and decode runs in the
CUDA library libkv2d.so.  PyTorch supplies device memory and streams.  If the
library is missing, every call raises; there is no fallback.
"""
from __future__ import annotations

import ctypes as C
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libkv2d.so")

KV2D_OK = 0
STATUS_NAMES = {0: "OK", 1: "INVALID_ARG", 2: "BUDGET_INFEASIBLE", 3: "WORKSPACE", 4: "CUDA",
                5: "DEVICE_FAULT", 6: "UNSUPPORTED", 7: "CAPACITY"}
FULL, TOK, CH, BOTH = 0, 1, 2, 3
OP_COMPRESS, OP_DECODE, OP_APPEND, OP_DECODE_SELECT = 0, 1, 2, 3
MAX_BATCH = 128


class Kv2dError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"kv2d {STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


class kv2d_params(C.Structure):
    _fields_ = [("head_dim", C.c_int32), ("num_q_heads", C.c_int32), ("num_kv_heads", C.c_int32),
                ("segment_len", C.c_int32), ("window", C.c_int32), ("keep_tokens", C.c_int32),
                ("keep_channels", C.c_int32), ("budget", C.c_float), ("scale", C.c_float),
                ("chunk_len", C.c_int32), ("chunk_budget", C.c_int32)]


class kv2d_dense(C.Structure):
    _fields_ = [("k", C.c_void_p), ("v", C.c_void_p), ("stride_b", C.c_int64),
                ("stride_h", C.c_int64), ("stride_t", C.c_int64), ("capacity", C.c_int32),
                ("block_table", C.c_void_p), ("block_size", C.c_int32), ("max_blocks", C.c_int32),
                ("num_blocks", C.c_int64)]


class kv2d_ccache(C.Structure):
    _fields_ = [("arena", C.c_void_p), ("arena_stride", C.c_int64), ("desc", C.c_void_p),
                ("max_segs", C.c_int32), ("n_segs", C.c_void_p), ("used_bytes", C.c_void_p),
                ("comp_end", C.c_void_p)]


class kv2d_staged(C.Structure):
    _fields_ = [("n_segs", C.c_void_p), ("used_bytes", C.c_void_p), ("comp_end", C.c_void_p)]


class kv2d_debug(C.Structure):
    _fields_ = [("a", C.c_void_p), ("lse", C.c_void_p), ("s", C.c_void_p), ("g", C.c_void_p),
                ("E", C.c_void_p), ("region_stride", C.c_int64), ("seg_stride", C.c_int32)]


EXPORTS = ["kv2d_segment_bytes", "kv2d_arena_bytes", "kv2d_workspace_bytes", "kv2d_compress",
           "kv2d_append", "kv2d_decode_attn", "kv2d_read_status", "kv2d_last_error",
           "kv2d_version", "kv2d_profile_enable", "kv2d_profile_read", "kv2d_set_decode_table_cap",
           "kv2d_profile_stage_name", "kv2d_decode_attn_noalloc", "kv2d_decode_attn_select",
           "kv2d_compress_staged", "kv2d_switch"]

_lib = None


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                               "python -m kv_cache_compression_kv2d_b200.build")
        L = C.CDLL(LIB_PATH)
        P = C.POINTER
        L.kv2d_segment_bytes.argtypes = [P(kv2d_params), C.c_int]
        L.kv2d_segment_bytes.restype = C.c_int64
        L.kv2d_arena_bytes.argtypes = [P(kv2d_params), C.c_int64]
        L.kv2d_arena_bytes.restype = C.c_int64
        L.kv2d_workspace_bytes.argtypes = [P(kv2d_params), C.c_int, C.c_int, C.c_int64]
        L.kv2d_workspace_bytes.restype = C.c_size_t
        L.kv2d_compress.argtypes = [P(kv2d_params), C.c_int, P(C.c_int32), P(C.c_int32),
                                    P(kv2d_dense), C.c_void_p, P(kv2d_ccache), C.c_void_p,
                                    C.c_size_t, P(kv2d_debug), C.c_void_p]
        L.kv2d_compress.restype = C.c_int
        L.kv2d_compress_staged.argtypes = [P(kv2d_params), C.c_int, P(C.c_int32), P(C.c_int32),
                                           P(kv2d_dense), C.c_void_p, P(kv2d_ccache),
                                           P(kv2d_staged), C.c_void_p, C.c_size_t, P(kv2d_debug),
                                           C.c_void_p]
        L.kv2d_compress_staged.restype = C.c_int
        L.kv2d_switch.argtypes = [P(kv2d_params), C.c_int, P(kv2d_ccache), P(kv2d_staged), C.c_void_p]
        L.kv2d_switch.restype = C.c_int
        L.kv2d_append.argtypes = [P(kv2d_params), C.c_int, P(kv2d_dense), C.c_void_p, C.c_void_p,
                                  C.c_void_p, C.c_void_p, C.c_size_t, C.c_void_p]
        L.kv2d_append.restype = C.c_int
        L.kv2d_decode_attn.argtypes = [P(kv2d_params), C.c_int, P(kv2d_ccache), P(kv2d_dense),
                                       C.c_void_p, C.c_int32, C.c_void_p, C.c_void_p, C.c_void_p,
                                       C.c_size_t, C.c_void_p]
        L.kv2d_decode_attn.restype = C.c_int
        L.kv2d_decode_attn_noalloc.argtypes = [P(kv2d_params), C.c_int, P(kv2d_ccache),
                                               P(kv2d_dense), C.c_void_p, C.c_int32, C.c_void_p,
                                               C.c_void_p, C.c_void_p, C.c_void_p]
        L.kv2d_decode_attn_noalloc.restype = C.c_int
        L.kv2d_decode_attn_select.argtypes = [P(kv2d_params), C.c_int, P(kv2d_ccache),
                                              P(kv2d_dense), C.c_void_p, C.c_int32, C.c_void_p,
                                              C.c_void_p, C.c_float, C.c_void_p, C.c_size_t,
                                              C.c_void_p, C.c_void_p, C.c_void_p]
        L.kv2d_decode_attn_select.restype = C.c_int
        L.kv2d_read_status.argtypes = [C.c_void_p, C.c_void_p, P(C.c_uint32)]
        L.kv2d_read_status.restype = C.c_int
        L.kv2d_last_error.argtypes = []
        L.kv2d_last_error.restype = C.c_char_p
        L.kv2d_version.argtypes = []
        L.kv2d_version.restype = C.c_char_p
        L.kv2d_set_decode_table_cap.argtypes = [C.c_int]
        L.kv2d_set_decode_table_cap.restype = C.c_int
        L.kv2d_profile_enable.argtypes = [C.c_int]
        L.kv2d_profile_enable.restype = C.c_int
        L.kv2d_profile_read.argtypes = [P(C.c_double), P(C.c_int64), C.c_int]
        L.kv2d_profile_read.restype = C.c_int
        L.kv2d_profile_stage_name.argtypes = [C.c_int]
        L.kv2d_profile_stage_name.restype = C.c_char_p
        _lib = L
    return _lib


# ------------------------------------------------------------- marshalling


def _ptr(t):
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream):
    if stream is None:
        if torch.cuda.is_available():
            return torch.cuda.current_stream().cuda_stream
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int):
    if rc != KV2D_OK:
        raise Kv2dError(rc, kv2d_last_error())
    return rc


def _i32_host(x, n):
    if isinstance(x, torch.Tensor):
        x = x.detach().cpu().tolist()
    arr = (C.c_int32 * n)(*[int(v) for v in list(x)[:n]])
    return arr


def params(head_dim, num_q_heads, num_kv_heads, segment_len, window, keep_tokens, keep_channels,
           budget, scale=0.0, chunk_len=0, chunk_budget=0) -> kv2d_params:
    return kv2d_params(int(head_dim), int(num_q_heads), int(num_kv_heads), int(segment_len),
                       int(window), int(keep_tokens), int(keep_channels), float(budget), float(scale),
                       int(chunk_len), int(chunk_budget))


def dense(k: torch.Tensor, v: torch.Tensor, block_table: torch.Tensor | None = None,
          block_size: int = 0) -> kv2d_dense:
    """Contiguous [B][Hkv][cap][d] tensors, or a paged pool
    [num_blocks][Hkv][block_size][d] with block_table [B][max_blocks]."""
    if block_table is None:
        return kv2d_dense(_ptr(k), _ptr(v), k.stride(0), k.stride(1), k.stride(2), k.shape[2],
                          None, 0, 0, 0)
    return kv2d_dense(_ptr(k), _ptr(v), 0, 0, 0, 0, _ptr(block_table), int(block_size),
                      block_table.shape[1], k.shape[0])


def kv2d_last_error() -> str:
    return lib().kv2d_last_error().decode()


def kv2d_version() -> str:
    return lib().kv2d_version().decode()


def kv2d_segment_bytes(p: kv2d_params, strategy: int) -> int:
    return int(lib().kv2d_segment_bytes(C.byref(p), int(strategy)))


def kv2d_arena_bytes(p: kv2d_params, max_tokens: int) -> int:
    return int(lib().kv2d_arena_bytes(C.byref(p), int(max_tokens)))


def kv2d_workspace_bytes(p: kv2d_params, op: int, batch: int, max_tokens: int) -> int:
    return int(lib().kv2d_workspace_bytes(C.byref(p), int(op), int(batch), int(max_tokens)))


def kv2d_compress(p, batch, seq_len_host, comp_end_host, dense_view, q_window, cc, ws,
                  dbg=None, stream=None, check=True) -> int:
    rc = lib().kv2d_compress(C.byref(p), int(batch), _i32_host(seq_len_host, batch),
                             _i32_host(comp_end_host, batch), C.byref(dense_view), _ptr(q_window),
                             C.byref(cc), _ptr(ws), ws.numel() if hasattr(ws, "numel") else 0,
                             C.byref(dbg) if dbg is not None else None, _stream(stream))
    return _check(rc) if check else rc


def kv2d_compress_staged(p, batch, seq_len_host, comp_end_host, dense_view, q_window, cc, staged,
                         ws, dbg=None, stream=None, check=True) -> int:
    """kv2d_compress whose bookkeeping goes to `staged` (a StagedRecord)
    until kv2d_switch publishes it."""
    rc = lib().kv2d_compress_staged(C.byref(p), int(batch), _i32_host(seq_len_host, batch),
                                    _i32_host(comp_end_host, batch), C.byref(dense_view),
                                    _ptr(q_window), C.byref(cc), C.byref(staged.struct), _ptr(ws),
                                    ws.numel() if hasattr(ws, "numel") else 0,
                                    C.byref(dbg) if dbg is not None else None, _stream(stream))
    return _check(rc) if check else rc


def kv2d_switch(p, batch, cc, staged, stream=None, check=True) -> int:
    """Publishes a staged compression as the cache's live bookkeeping."""
    rc = lib().kv2d_switch(C.byref(p), int(batch), C.byref(cc), C.byref(staged.struct),
                           _stream(stream))
    return _check(rc) if check else rc


def kv2d_append(p, batch, dense_view, k_new, v_new, seq_len_dev, ws, stream=None,
                check=True) -> int:
    rc = lib().kv2d_append(C.byref(p), int(batch), C.byref(dense_view), _ptr(k_new), _ptr(v_new),
                           _ptr(seq_len_dev), _ptr(ws), ws.numel() if hasattr(ws, "numel") else 0,
                           _stream(stream))
    return _check(rc) if check else rc


def kv2d_decode_attn(p, batch, cc, dense_view, seq_len_dev, max_seq_len_host, q, out, ws,
                     stream=None, check=True) -> int:
    rc = lib().kv2d_decode_attn(C.byref(p), int(batch), C.byref(cc), C.byref(dense_view),
                                _ptr(seq_len_dev), int(max_seq_len_host), _ptr(q), _ptr(out),
                                _ptr(ws), ws.numel() if hasattr(ws, "numel") else 0,
                                _stream(stream))
    return _check(rc) if check else rc


def kv2d_decode_attn_select(p, batch, cc, dense_view, seq_len_dev, max_seq_len_host, q, out,
                            select_rate, ws, dbg_score=None, dbg_sel=None, stream=None,
                            check=True) -> int:
    """Decode attention with decode-time token selection at select_rate
    (dbg_score / dbg_sel: optional per-slot scores and kept flags)."""
    rc = lib().kv2d_decode_attn_select(C.byref(p), int(batch), C.byref(cc), C.byref(dense_view),
                                       _ptr(seq_len_dev), int(max_seq_len_host), _ptr(q),
                                       _ptr(out), float(select_rate), _ptr(ws),
                                       ws.numel() if hasattr(ws, "numel") else 0, _ptr(dbg_score),
                                       _ptr(dbg_sel), _stream(stream))
    return _check(rc) if check else rc


def kv2d_set_decode_table_cap(cap: int) -> None:
    """Testing aid: blocks per chunk of the decode kernel's block table
    (0 restores the default)."""
    _check(lib().kv2d_set_decode_table_cap(int(cap)))


def kv2d_profile_enable(on: bool) -> int:
    return int(lib().kv2d_profile_enable(1 if on else 0))


def kv2d_profile_read() -> dict:
    """{stage name: (total ms, launches)} since the last read."""
    ms = (C.c_double * 32)()
    n_l = (C.c_int64 * 32)()
    n = lib().kv2d_profile_read(ms, n_l, 32)
    out = {}
    for i in range(n):
        out[lib().kv2d_profile_stage_name(i).decode()] = (float(ms[i]), int(n_l[i]))
    return out


def kv2d_decode_attn_noalloc(p, batch, cc, dense_view, seq_len_dev, max_seq_len_host, q, out,
                             status_dev=None, stream=None, check=True) -> int:
    """kv2d_decode_attn without a workspace: for callers that cannot allocate
    device memory (scratch is the library's fixed per-GPU array)."""
    rc = lib().kv2d_decode_attn_noalloc(C.byref(p), int(batch), C.byref(cc), C.byref(dense_view),
                                        _ptr(seq_len_dev), int(max_seq_len_host), _ptr(q),
                                        _ptr(out), _ptr(status_dev), _stream(stream))
    return _check(rc) if check else rc


def kv2d_read_status(ws, stream=None) -> int:
    bits = C.c_uint32(0)
    lib().kv2d_read_status(_ptr(ws), _stream(stream), C.byref(bits))
    return int(bits.value)


# ------------------------------------------------ caller-owned buffers


class CompressedCache:
    """Device buffers of one layer's compressed cache (caller-owned memory,
    allocated through torch) and the kv2d_ccache struct that points at them."""

    def __init__(self, p: kv2d_params, batch: int, max_tokens: int, device="cuda"):
        units = batch * p.num_kv_heads
        self.arena_stride = kv2d_arena_bytes(p, max_tokens)
        if self.arena_stride < 0:
            raise Kv2dError(1, "invalid params")
        self.max_segs = max(1, max_tokens // p.segment_len)
        self.arena = torch.zeros(units * self.arena_stride, dtype=torch.uint8, device=device)
        self.desc = torch.zeros((units, self.max_segs), dtype=torch.int64, device=device)
        # bookkeeping in one buffer: used_bytes (int64), then n_segs and
        # comp_end (int32), so that reset() is a single fill
        n32 = units + batch
        self.book = torch.zeros(units + (n32 + 1) // 2, dtype=torch.int64, device=device)
        self.used_bytes = self.book[:units]
        book32 = self.book[units:].view(torch.int32)
        self.n_segs = book32[:units]
        self.comp_end = book32[units:units + batch]
        self.struct = kv2d_ccache(_ptr(self.arena), self.arena_stride, _ptr(self.desc),
                                  self.max_segs, _ptr(self.n_segs), _ptr(self.used_bytes),
                                  _ptr(self.comp_end))

    def reset(self):
        """Forget every compressed segment (the arena bytes are left as they
        are; descriptors past n_segs are never read)."""
        self.book.zero_()


class StagedRecord:
    """Device buffers of a staged compression's bookkeeping (caller-owned)."""

    def __init__(self, p: kv2d_params, batch: int, device="cuda"):
        units = batch * p.num_kv_heads
        self.used_bytes = torch.zeros(units, dtype=torch.int64, device=device)
        self.n_segs = torch.zeros(units, dtype=torch.int32, device=device)
        self.comp_end = torch.zeros(batch, dtype=torch.int32, device=device)
        self.struct = kv2d_staged(_ptr(self.n_segs), _ptr(self.used_bytes), _ptr(self.comp_end))


def workspace(nbytes: int, device="cuda") -> torch.Tensor:
    """Zeroed scratch buffer (torch allocations are 512-byte aligned)."""
    return torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device)
