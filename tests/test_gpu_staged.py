"""Compression that does not block decode: kv2d_compress_staged on a second
stream while decode steps (append + decode) go on in the decode stream, then
kv2d_switch on the decode stream.  Before the switch every decode equals the
oracle's decode over the old segments plus the dense tail (which still holds
the tokens being compressed); after it, over the new segments; and the
published cache equals, byte for byte, what a plain kv2d_compress of the same
region writes."""
import numpy as np
import pytest
import torch

from kv_cache_compression_kv2d_b200 import binding as B
from kv_cache_compression_kv2d_b200 import synth
from kv_cache_compression_kv2d_b200.synth import Workload

from tests import gpu_harness as H

pytestmark = pytest.mark.gpu

WL = Workload("staged", 3, 2, 4, 128, 1537, 64, 32, 0.3, ragged_min=700)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from kv_cache_compression_kv2d_b200 import build
    build.build()
    assert torch.cuda.is_available()
    B.lib()


def _decode_matches(orc, run, q):
    out = H.gpu_decode(run, q).float().cpu().numpy()
    G = WL.group
    for b in range(WL.batch):
        for h in range(WL.num_kv_heads):
            ref = H.oracle_decode_unit(orc, run, b, h, q)
            err = float(np.max(np.abs(out[b, h * G:(h + 1) * G] - ref)))
            assert err <= H.TOL_OUT, f"decode unit ({b}, {h}): {err}"


def _runs():
    host = synth.generate(WL, seed=3, extra_capacity=200)
    runs = [H.make_run(WL, H.to_device(host), H.params_for(WL)) for _ in range(2)]
    for run in runs:
        H.compress(run)
    return runs


def test_staged_compress_then_switch(orc):
    run, plain = _runs()
    ws_a = B.workspace(256)
    # 100 decode steps in both copies: new complete segments appear
    for step in range(100):
        k, v, _ = synth.decode_tokens(WL, step, seed=3, device="cuda", mu=run.batch.mu)
        for r in (run, plain):
            B.kv2d_append(r.p, WL.batch, r.dv, k, v, r.seq_len, ws_a)
    torch.cuda.synchronize()
    seq_host = run.seq_len.cpu().tolist()
    ce_old = run.cc.comp_end.cpu().tolist()
    n_old = run.cc.n_segs.clone()
    used_old = run.cc.used_bytes.clone()

    # reference: a plain compression of the same region in the second copy
    H.compress(plain, seq_host=seq_host)

    # staged compression on a side stream, decode steps meanwhile
    staged = B.StagedRecord(run.p, WL.batch)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    ws_c = B.workspace(B.kv2d_workspace_bytes(run.p, B.OP_COMPRESS, WL.batch, max(seq_host)))
    with torch.cuda.stream(side):
        B.kv2d_compress_staged(run.p, WL.batch, seq_host, ce_old, run.dv, run.batch.qw,
                               run.cc.struct, staged, ws_c, stream=side)
        done = torch.cuda.Event()
        done.record(side)
    for step in range(100, 103):
        k, v, q = synth.decode_tokens(WL, step, seed=3, device="cuda", mu=run.batch.mu)
        B.kv2d_append(run.p, WL.batch, run.dv, k, v, run.seq_len, ws_a)
        B.kv2d_append(plain.p, WL.batch, plain.dv, k, v, plain.seq_len, ws_a)
        # the live bookkeeping is the old one whatever the side stream has done
        assert torch.equal(run.cc.n_segs, n_old) and torch.equal(run.cc.used_bytes, used_old)
        _decode_matches(orc, run, q)
    torch.cuda.current_stream().wait_event(done)
    B.kv2d_switch(run.p, WL.batch, run.cc.struct, staged)
    torch.cuda.synchronize()
    assert B.kv2d_read_status(ws_c) == 0
    # published: bookkeeping, descriptors and packed bytes equal the plain compression
    assert torch.equal(run.cc.n_segs, plain.cc.n_segs)
    assert torch.equal(run.cc.used_bytes, plain.cc.used_bytes)
    assert torch.equal(run.cc.comp_end, plain.cc.comp_end)
    assert int((run.cc.n_segs - n_old).sum()) > 0, "the staged call compressed nothing"
    units = WL.batch * WL.num_kv_heads
    for u in range(units):
        n = int(run.cc.n_segs[u])
        used = int(run.cc.used_bytes[u])
        assert torch.equal(run.cc.desc[u, :n], plain.cc.desc[u, :n])
        s = u * run.cc.arena_stride
        assert torch.equal(run.cc.arena[s:s + used], plain.cc.arena[s:s + used])
    _, _, q = synth.decode_tokens(WL, 103, seed=3, device="cuda", mu=run.batch.mu)
    _decode_matches(orc, run, q)


def test_staged_without_new_segments_keeps_the_live_values(orc):
    run, _ = _runs()
    seq_host = run.seq_len.cpu().tolist()
    ce = run.cc.comp_end.cpu().tolist()
    before = (run.cc.n_segs.clone(), run.cc.used_bytes.clone(), run.cc.comp_end.clone())
    staged = B.StagedRecord(run.p, WL.batch)
    staged.n_segs.fill_(-5)
    ws_c = B.workspace(B.kv2d_workspace_bytes(run.p, B.OP_COMPRESS, WL.batch, max(seq_host)))
    B.kv2d_compress_staged(run.p, WL.batch, seq_host, ce, run.dv, run.batch.qw, run.cc.struct,
                           staged, ws_c)
    B.kv2d_switch(run.p, WL.batch, run.cc.struct, staged)
    torch.cuda.synchronize()
    assert torch.equal(run.cc.n_segs, before[0])
    assert torch.equal(run.cc.used_bytes, before[1])
    assert torch.equal(run.cc.comp_end, before[2])
