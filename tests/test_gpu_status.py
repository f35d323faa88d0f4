"""Device-side faults are reported through the status word, not by trapping.

Inputs that only the device can see to be wrong -- a block-table entry that
points past the block pool, a device sequence length past the view's
capacity -- are made on the host and handed to compress, append and decode.
Each kernel's own bounds check skips the access and ORs the documented bit
(KV2D_DEV_BLOCK_TABLE, KV2D_DEV_SEQ_RANGE) into the status word, which
kv2d_read_status returns.  The sequences that were not touched still match
the oracle.  Every bad index here is caught by a check in the kernel before
any load or store uses it: the TMA key loads substitute block 0, the row
helpers return no row, and decode clamps the lengths it reads.
"""
import numpy as np
import pytest
import torch

from kv_cache_compression_kv2d_b200 import binding as B
from kv_cache_compression_kv2d_b200 import synth
from kv_cache_compression_kv2d_b200.synth import Workload

from tests import gpu_harness as H

pytestmark = pytest.mark.gpu

DEV_BLOCK_TABLE, DEV_SEQ_RANGE = 1, 8
WL = Workload("status_paged", 3, 2, 4, 128, 1400, 64, 32, 0.25, ragged_min=600, block_size=16)


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from kv_cache_compression_kv2d_b200 import build
    build.build()
    assert torch.cuda.is_available()
    B.lib()


def _run():
    host = synth.generate(WL, seed=5, extra_capacity=40)
    return H.make_run(WL, H.to_device(host), H.params_for(WL))


def test_block_table_out_of_range_in_compress(orc):
    run = _run()
    bt = run.batch.block_table
    nblocks = run.batch.k.shape[0]
    good = int(bt[1, 5])
    bt[1, 5] = nblocks                      # a block inside sequence 1's first segments
    torch.cuda.synchronize()
    H.compress(run, expect_bits=DEV_BLOCK_TABLE)
    bt[1, 5] = good
    for b in (0, 2):
        for h in range(WL.num_kv_heads):
            H.check_compress_unit(orc, run, b, h, independent=True)
    q = run.batch.q
    out = H.gpu_decode(run, q).float().cpu().numpy()
    G = WL.group
    for b in (0, 2):
        for h in range(WL.num_kv_heads):
            ref = H.oracle_decode_unit(orc, run, b, h, q)
            assert float(np.max(np.abs(out[b, h * G:(h + 1) * G] - ref))) <= H.TOL_OUT


def test_block_table_out_of_range_in_decode(orc):
    run = _run()
    H.compress(run)
    seq = run.seq_len.cpu().tolist()
    ce = run.cc.comp_end.cpu().tolist()
    # a sequence with a dense tail: its last block is read by decode only
    b_bad = next(b for b in range(WL.batch) if seq[b] > ce[b])
    bt = run.batch.block_table
    blk = (seq[b_bad] - 1) // WL.block_size
    good = int(bt[b_bad, blk])
    bt[b_bad, blk] = run.batch.k.shape[0] + 7
    torch.cuda.synchronize()
    q = run.batch.q
    out = H.gpu_decode(run, q, expect_bits=DEV_BLOCK_TABLE).float().cpu().numpy()
    bt[b_bad, blk] = good
    assert np.isfinite(out).all()
    G = WL.group
    for b in range(WL.batch):
        if b == b_bad:
            continue
        for h in range(WL.num_kv_heads):
            ref = H.oracle_decode_unit(orc, run, b, h, q)
            assert float(np.max(np.abs(out[b, h * G:(h + 1) * G] - ref))) <= H.TOL_OUT


def test_sequence_length_out_of_range_in_append_and_decode(orc):
    run = _run()
    H.compress(run)
    cap = run.dv.max_blocks * run.dv.block_size
    seq0 = run.seq_len.cpu().tolist()
    # append: sequence 2 is full (its next row would be row `cap`)
    run.seq_len[2] = cap
    k, v, q = synth.decode_tokens(WL, 0, seed=5, device="cuda", mu=run.batch.mu)
    ws = B.workspace(256)
    B.kv2d_append(run.p, WL.batch, run.dv, k, v, run.seq_len, ws)
    torch.cuda.synchronize()
    assert B.kv2d_read_status(ws) == DEV_SEQ_RANGE
    seq1 = run.seq_len.cpu().tolist()
    assert seq1 == [seq0[0] + 1, seq0[1] + 1, cap]
    for b in (0, 1):
        for h in range(WL.num_kv_heads):
            kr, vr = synth.dense_rows(run.batch, b, h, seq0[b], seq0[b] + 1)
            assert torch.equal(kr[0], k[b, h]) and torch.equal(vr[0], v[b, h])
    # decode: sequence 2 claims more tokens than the view holds
    run.seq_len[2] = cap + 5
    out = H.gpu_decode(run, q, max_seq=cap, expect_bits=None)
    ws_bits = _decode_bits(run, q, cap)
    assert ws_bits & DEV_SEQ_RANGE
    out = out.float().cpu().numpy()
    G = WL.group
    for b in (0, 1):
        for h in range(WL.num_kv_heads):
            ref = H.oracle_decode_unit(orc, run, b, h, q)
            assert float(np.max(np.abs(out[b, h * G:(h + 1) * G] - ref))) <= H.TOL_OUT
    run.seq_len[2] = seq0[2]


def _decode_bits(run, q, cap):
    out = torch.empty((WL.batch, WL.num_q_heads, WL.head_dim), dtype=torch.float16, device="cuda")
    ws = B.workspace(B.kv2d_workspace_bytes(run.p, B.OP_DECODE, WL.batch, cap))
    B.kv2d_decode_attn(run.p, WL.batch, run.cc.struct, run.dv, run.seq_len, cap, q, out, ws)
    torch.cuda.synchronize()
    bits = B.kv2d_read_status(ws)
    assert B.kv2d_read_status(ws) == 0      # reading clears the word
    return bits
