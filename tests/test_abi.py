"""The C-ABI library loads, exports every symbol include/kv2d.h declares, and
rejects bad arguments on the host with the documented status codes before
any CUDA call (these tests run without a GPU)."""
import ctypes as C
import os
import re

import numpy as np
import pytest

from kv_cache_compression_kv2d_b200 import binding as B
from kv_cache_compression_kv2d_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    kbuild.build()
    return B.lib()


def test_exports_match_header(L):
    with open(os.path.join(ROOT, "include", "kv2d.h")) as f:
        hdr = f.read()
    declared = re.findall(r"KV2D_API\s+[\w\s\*]+?\b(kv2d_\w+)\s*\(", hdr)
    assert len(declared) >= 9
    assert sorted(declared) == sorted(B.EXPORTS)
    for name in declared:
        assert hasattr(L, name), name
    assert B.kv2d_version().startswith("kv2d")


def test_segment_bytes_agree_with_oracle(L, orc):
    for (S, r, c) in [(64, 8, 32), (128, 16, 32), (16, 3, 5), (256, 32, 128), (48, 48, 1)]:
        p = B.params(128, 32, 8, S, 16, r, c, 0.2)
        po = orc.params(128, 4, S, 16, r, c, 0.2)
        for st in range(4):
            assert B.kv2d_segment_bytes(p, st) == orc.segment_bytes(po, st)
        assert B.kv2d_segment_bytes(p, 4) == -1


def test_arena_bound_covers_budget(L, orc):
    for beta in (0.1, 0.15, 0.2, 0.25, 1.0, 1.7):
        p = B.params(128, 32, 8, 64, 64, 8, 32, beta)
        po = orc.params(128, 4, 64, 64, 8, 32, beta)
        for T in (0, 63, 64, 4096, 32768, 131072 + 17):
            nb = B.kv2d_arena_bytes(p, T)
            assert nb % 256 == 0
            nseg = T // 64
            most = nseg * 32768 if beta >= 1 else orc.budget_bytes(
                orc.params(128, 4, 64, 64, 8, 32, float(np.float32(beta))), nseg)
            assert nb >= most


def test_workspace_sizes(L):
    p = B.params(128, 32, 8, 64, 64, 8, 32, 0.2)
    a = B.kv2d_workspace_bytes(p, B.OP_COMPRESS, 1, 32768)
    b = B.kv2d_workspace_bytes(p, B.OP_COMPRESS, 2, 32768)
    assert 0 < a < b and a % 256 == 0
    assert B.kv2d_workspace_bytes(p, B.OP_DECODE, 16, 131072) > 0
    assert B.kv2d_workspace_bytes(p, B.OP_APPEND, 1, 0) == 256
    assert B.kv2d_workspace_bytes(p, 9, 1, 10) == 0
    assert B.kv2d_workspace_bytes(p, B.OP_COMPRESS, 0, 10) == 0
    assert B.kv2d_workspace_bytes(p, B.OP_COMPRESS, B.MAX_BATCH + 1, 10) == 0


def _fake_dense(T=4096, Hkv=8, d=128):
    # host-side validation only: aligned fake device addresses, never dereferenced
    return B.kv2d_dense(1 << 20, 2 << 20, Hkv * T * d, T * d, d, T, None, 0, 0, 0)


def _fake_cc(max_segs=1 << 12, stride=1 << 24):
    return B.kv2d_ccache(3 << 20, stride, 4 << 20, max_segs, 5 << 20, 6 << 20, 7 << 20)


def _compress(p, batch, seq, ce, dense=None, cc=None, ws_bytes=1 << 30, q=8 << 20):
    n = max(batch, 1)
    seq_a = (C.c_int32 * n)(*seq)
    ce_a = (C.c_int32 * n)(*ce)
    d = dense or _fake_dense()
    c = cc or _fake_cc()
    return B.lib().kv2d_compress(C.byref(p), batch, seq_a, ce_a, C.byref(d), q, C.byref(c),
                                 9 << 20, ws_bytes, None, None)


@pytest.mark.parametrize("field,value,code", [
    ("head_dim", 96, 1), ("head_dim", 64, 6), ("segment_len", 72, 1), ("segment_len", 512, 1),
    ("window", 0, 1), ("window", 129, 1), ("keep_tokens", 0, 1), ("keep_tokens", 65, 1),
    ("keep_channels", 129, 1), ("keep_channels", 0, 1), ("budget", 0.0, 1),
    ("budget", float("nan"), 1), ("num_kv_heads", 3, 1), ("scale", -1.0, 1),
    ("chunk_len", 2, 1), ("chunk_len", 65, 1), ("chunk_len", -1, 1),
])
def test_invalid_params_rejected(L, field, value, code):
    p = B.params(128, 32, 8, 64, 64, 8, 32, 0.2)
    setattr(p, field, value)
    assert _compress(p, 1, [4096], [0]) == code
    assert B.kv2d_last_error() != ""


def test_host_checks(L):
    p = B.params(128, 32, 8, 64, 64, 8, 32, 0.2)
    assert _compress(p, 0, [4096], [0]) == 1                      # batch
    assert _compress(p, 1, [5000], [0]) == 1                      # beyond capacity
    assert _compress(p, 1, [4096], [32]) == 1                     # comp_end not multiple of S
    # window (64) longer than the region (100 - 64 = 36 tokens)? region 100 -> 1 segment
    pw = B.params(128, 32, 8, 64, 128, 8, 32, 0.2)
    assert _compress(pw, 1, [100], [0]) == 1
    # budget infeasible: 8% < cheapest (BOTH, 8.64%)
    pb = B.params(128, 32, 8, 64, 64, 8, 32, 0.08)
    assert _compress(pb, 1, [4096], [0]) == 2
    # descriptor table too small
    assert _compress(p, 1, [4096], [0], cc=_fake_cc(max_segs=10)) == 7
    # arena too small
    assert _compress(p, 1, [4096], [0], cc=_fake_cc(stride=256)) == 7
    # misaligned arena stride
    assert _compress(p, 1, [4096], [0], cc=_fake_cc(stride=1000)) == 1
    # unaligned dense pointer
    d = _fake_dense()
    d.k = (1 << 20) + 8
    assert _compress(p, 1, [4096], [0], dense=d) == 1
    # workspace too small
    assert _compress(p, 1, [4096], [0], ws_bytes=1024) == 3
    # nothing complete to compress: OK without any launch
    assert _compress(p, 1, [63], [0]) == 0


def test_decode_and_append_host_checks(L):
    p = B.params(128, 32, 8, 64, 64, 8, 32, 0.2)
    d = _fake_dense()
    cc = _fake_cc()
    lib = B.lib()
    # G = 1 decode is not built
    p1 = B.params(128, 8, 8, 64, 64, 8, 32, 0.2)
    assert lib.kv2d_decode_attn(C.byref(p1), 1, C.byref(cc), C.byref(d), 1 << 22, 4096,
                                1 << 23, 1 << 24, 9 << 20, 1 << 30, None) == 6
    # max_seq_len beyond capacity
    assert lib.kv2d_decode_attn(C.byref(p), 1, C.byref(cc), C.byref(d), 1 << 22, 5000,
                                1 << 23, 1 << 24, 9 << 20, 1 << 30, None) == 1
    # workspace too small
    assert lib.kv2d_decode_attn(C.byref(p), 1, C.byref(cc), C.byref(d), 1 << 22, 4096,
                                1 << 23, 1 << 24, 9 << 20, 64, None) == 3
    # append: NULL new token
    assert lib.kv2d_append(C.byref(p), 1, C.byref(d), None, 1 << 23, 1 << 22, 9 << 20, 256,
                           None) == 1
    # paged view with a block size that is not a multiple of 16
    dp = B.kv2d_dense(1 << 20, 2 << 20, 0, 0, 0, 0, 1 << 21, 8, 16, 100)
    assert lib.kv2d_append(C.byref(p), 1, C.byref(dp), 1 << 23, 1 << 23, 1 << 22, 9 << 20, 256,
                           None) == 1


def test_cache_bookkeeping_views_and_reset(L):
    """n_segs, used_bytes and comp_end live in one buffer: writing one never
    touches another, and reset() clears all three with one fill."""
    import torch
    p = B.params(128, 32, 8, 64, 64, 8, 32, 0.2)
    cc = B.CompressedCache(p, 3, 4096, device="cpu")
    assert cc.n_segs.dtype == torch.int32 and cc.n_segs.numel() == 24
    assert cc.used_bytes.dtype == torch.int64 and cc.used_bytes.numel() == 24
    assert cc.comp_end.dtype == torch.int32 and cc.comp_end.numel() == 3
    cc.used_bytes.copy_(torch.arange(24, dtype=torch.int64) + (1 << 40))
    cc.n_segs.copy_(torch.arange(24, dtype=torch.int32) + 7)
    cc.comp_end.copy_(torch.tensor([64, 128, 192], dtype=torch.int32))
    assert torch.equal(cc.used_bytes, torch.arange(24, dtype=torch.int64) + (1 << 40))
    assert torch.equal(cc.n_segs, torch.arange(24, dtype=torch.int32) + 7)
    assert cc.comp_end.tolist() == [64, 128, 192]
    ptrs = [cc.used_bytes.data_ptr(), cc.n_segs.data_ptr(), cc.comp_end.data_ptr()]
    assert all(x % 4 == 0 for x in ptrs) and ptrs[0] % 8 == 0
    cc.reset()
    assert int(cc.used_bytes.abs().sum()) == 0
    assert int(cc.n_segs.abs().sum()) == 0 and int(cc.comp_end.abs().sum()) == 0


def test_decode_table_cap_range(L):
    # host-only setter: 0 (default) or [32, 4096]
    for bad in (31, 4097, -1):
        with pytest.raises(B.Kv2dError):
            B.kv2d_set_decode_table_cap(bad)
    for good in (32, 4096, 0):
        B.kv2d_set_decode_table_cap(good)


def test_noalloc_decode_rejects_oversize_before_launch(L):
    """The scratch-array decode refuses, on the host, a shape whose scratch
    would not fit its fixed array (8 MiB): 128 sequences x 64 KV heads with 8
    query heads each need (8192 units + CTAs) x 8 x 132 x 4 bytes, about
    35 MB.  The check runs before any CUDA call, so the fake pointers are
    never used."""
    lib = B.lib()
    d = B.kv2d_dense(1 << 20, 2 << 20, 64 * 4096 * 128, 4096 * 128, 128, 4096, None, 0, 0, 0)
    cc = _fake_cc()
    big = B.params(128, 512, 64, 64, 64, 8, 32, 0.2)
    rc = lib.kv2d_decode_attn_noalloc(C.byref(big), 128, C.byref(cc), C.byref(d), 1 << 22, 4096,
                                      1 << 23, 1 << 24, None, None)
    assert rc == 3
    assert "scratch" in B.kv2d_last_error()


def test_chunk_params_checked(L):
    """Token2Chunk needs 1 <= chunk_budget < r when chunk_len is set, and at
    most 33 core tokens; chunk_budget is ignored when chunk_len is 0."""
    for (r, alpha, code) in [(8, 0, 1), (8, 8, 1), (8, 4, 0), (40, 6, 6), (40, 7, 0)]:
        p = B.params(128, 32, 8, 64, 64, r, 32, 0.2, chunk_len=8, chunk_budget=alpha)
        rc = _compress(p, 1, [63], [0])          # nothing complete: OK without a launch
        assert rc == code, (r, alpha, rc)
    p = B.params(128, 32, 8, 64, 64, 8, 32, 0.2, chunk_len=0, chunk_budget=99)
    assert _compress(p, 1, [63], [0]) == 0


def test_switch_and_staged_host_checks(L):
    """The staged compression and the switch reject a missing staged record,
    an out-of-range batch and NULL bookkeeping pointers on the host, before
    anything is launched (the fake addresses are never used)."""
    lib = B.lib()
    p = B.params(128, 32, 8, 64, 64, 8, 32, 0.2)
    cc = _fake_cc()
    st = B.kv2d_staged(8 << 20, 9 << 20, 10 << 20)
    assert lib.kv2d_switch(C.byref(p), 1, C.byref(cc), None, None) == 1
    assert lib.kv2d_switch(C.byref(p), 0, C.byref(cc), C.byref(st), None) == 1
    assert lib.kv2d_switch(C.byref(p), 129, C.byref(cc), C.byref(st), None) == 1
    assert lib.kv2d_switch(C.byref(p), 1, C.byref(cc), C.byref(B.kv2d_staged(None, 9 << 20, 10 << 20)),
                           None) == 1
    cc0 = B.kv2d_ccache(3 << 20, 1 << 24, 4 << 20, 1 << 12, None, 6 << 20, 7 << 20)
    assert lib.kv2d_switch(C.byref(p), 1, C.byref(cc0), C.byref(st), None) == 1
    bad = B.params(128, 30, 8, 64, 64, 8, 32, 0.2)          # Hq not a multiple of Hkv
    assert lib.kv2d_switch(C.byref(bad), 1, C.byref(cc), C.byref(st), None) == 1
    seq = (C.c_int32 * 1)(4096)
    ce = (C.c_int32 * 1)(0)
    d = _fake_dense()
    assert lib.kv2d_compress_staged(C.byref(p), 1, seq, ce, C.byref(d), 8 << 20, C.byref(cc), None,
                                    9 << 20, 1 << 30, None, None) == 1
    assert "staged" in B.kv2d_last_error()


def test_select_decode_host_checks(L):
    """The selection decode rejects a non-positive or non-finite rate, a
    group wider than 8 and a length beyond the capacity on the host, before
    anything is launched."""
    lib = B.lib()
    p = B.params(128, 32, 8, 64, 64, 8, 32, 0.2)
    cc = _fake_cc()
    d = _fake_dense()
    args = (1 << 22, 4096, 1 << 23, 1 << 24)
    for rate in (0.0, -0.1, float("nan"), float("inf")):
        assert lib.kv2d_decode_attn_select(C.byref(p), 1, C.byref(cc), C.byref(d), *args, rate,
                                           9 << 20, 1 << 30, None, None, None) == 1
    assert lib.kv2d_decode_attn_select(C.byref(p), 1, C.byref(cc), C.byref(d), 1 << 22, 5000,
                                       1 << 23, 1 << 24, 0.1, 9 << 20, 1 << 30, None, None, None) == 1
    wide = B.params(128, 128, 8, 64, 16, 8, 32, 0.2)        # G = 16
    assert lib.kv2d_decode_attn_select(C.byref(wide), 1, C.byref(cc), C.byref(d), *args, 0.1,
                                       9 << 20, 1 << 30, None, None, None) == 6
