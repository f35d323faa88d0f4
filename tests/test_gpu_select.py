"""Decode with decode-time token selection (MosaicKV stage 2) against the
oracle, per unit:
  1. the candidate scores against the oracle's fp64 scores (relative 1e-4,
     absolute floor 1: they are logits);
  2. the oracle fed the GPU's fp32 scores picks the same slots, bit for bit
     (ties to the lower slot);
  3. the output against the oracle's attention over those slots and the
     dense tail: max abs error <= 2e-3;
  4. the fully independent oracle (its own fp64 scores and choice): the share
     of kept slots both pick, and its output difference, are printed and
     bounded.
A rate that keeps every candidate equals the plain decode."""
import numpy as np
import pytest
import torch

from kv_cache_compression_kv2d_b200 import binding as B
from kv_cache_compression_kv2d_b200 import synth
from kv_cache_compression_kv2d_b200.synth import Workload

from tests import gpu_harness as H

pytestmark = pytest.mark.gpu

CASES = {
    "ragged_multi": Workload("ragged_multi", 3, 2, 4, 128, 1537, 64, 24, 0.3, ragged_min=700),
    "paged": Workload("paged", 3, 2, 4, 128, 1400, 64, 32, 0.25, ragged_min=600, block_size=16),
    "mix4": Workload("mix4", 2, 2, 4, 128, 2048, 64, 64, 0.15, segment_mix=True),
    "g8_gw384": Workload("g8_gw384", 2, 1, 8, 128, 1100, 32, 48, 0.3),
    "g2_small_rc": Workload("g2_small_rc", 2, 2, 2, 128, 999, 16, 64, 0.35, keep_tokens=3,
                            keep_channels=20),
    "gw512_s128": Workload("gw512_s128", 1, 2, 4, 128, 2048 + 77, 128, 128, 0.15),
}
MIN_AGREEMENT = 0.98
TOL_END_TO_END = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from kv_cache_compression_kv2d_b200 import build
    build.build()
    assert torch.cuda.is_available()
    B.lib()


def _run(wl, seed=0, **kw):
    batch = synth.generate(wl, seed=seed, device="cpu", extra_capacity=4)
    run = H.make_run(wl, H.to_device(batch), H.params_for(wl, **kw))
    H.compress(run)
    return run


def check_select(orc, run, rate, units=None, label=""):
    wl = run.wl
    po = H.oracle_params(orc, run.p)
    q = run.batch.q
    out, score, sel = H.gpu_decode_select(run, q, rate)
    out = out.float().cpu().numpy()
    score = score.cpu().numpy()
    sel = sel.cpu().numpy()
    G, S = wl.group, wl.segment_len
    rate32 = float(np.float32(rate))
    units = units or [(b, h) for b in range(wl.batch) for h in range(wl.num_kv_heads)]
    agree = total = 0
    worst_e2e = 0.0
    for b, h in units:
        u = b * wl.num_kv_heads + h
        arena, offs, strat, Kt, Vt = H.unit_cache(run, b, h)
        nslot = len(strat) * S
        qh = q[b, h * G:(h + 1) * G].cpu().numpy()
        ref_score, ncand = orc.select_scores(po, arena, offs, strat, qh)
        gs = score[u, :nslot].astype(np.float64)
        assert np.array_equal(np.isinf(gs), np.isinf(ref_score)), "candidate slots differ"
        fin = np.isfinite(ref_score)
        err = np.abs(gs[fin] - ref_score[fin]) / np.maximum(1.0, np.abs(ref_score[fin]))
        assert err.size == 0 or np.max(err) < H.TOL_REL, f"score mismatch {np.max(err)}"
        n_sel = orc.select_count(po, len(strat), ncand, rate32)
        fed = orc.select_tokens(gs, n_sel)
        assert np.array_equal(sel[u, :nslot], fed), f"unit ({b}, {h}): selection differs"
        o_ref = orc.decode_select(po, arena, offs, strat, fed, Kt, Vt, qh)
        e = float(np.max(np.abs(out[b, h * G:(h + 1) * G] - o_ref)))
        assert e <= H.TOL_OUT, f"unit ({b}, {h}): output error {e}"
        own = orc.select_tokens(ref_score, n_sel)
        agree += int(np.sum(own.astype(bool) & fed.astype(bool)))
        total += n_sel
        o_own = orc.decode_select(po, arena, offs, strat, own, Kt, Vt, qh)
        worst_e2e = max(worst_e2e, float(np.max(np.abs(out[b, h * G:(h + 1) * G] - o_own))))
    frac = agree / max(total, 1)
    print(f"\nSELECT {label} rate {rate}: kept-slot agreement {agree}/{total} = {frac:.4f}, "
          f"independent output difference {worst_e2e:.3e}")
    assert frac >= MIN_AGREEMENT
    assert worst_e2e <= TOL_END_TO_END


@pytest.mark.parametrize("name", list(CASES))
@pytest.mark.parametrize("rate", [0.0625, 0.125])
def test_select_decode_parity(orc, name, rate):
    run = _run(CASES[name])
    check_select(orc, run, rate, label=name)


def test_select_after_append_and_periodic_compress(orc):
    wl = CASES["ragged_multi"]
    run = _run(wl)
    ws = B.workspace(256)
    for step in range(70):
        k, v, q = synth.decode_tokens(wl, step, device="cuda", mu=run.batch.mu)
        B.kv2d_append(run.p, wl.batch, run.dv, k, v, run.seq_len, ws)
    torch.cuda.synchronize()
    H.compress(run, seq_host=run.seq_len.cpu().tolist())
    run.batch = run.batch.__class__(**{**run.batch.__dict__, "q": q})
    check_select(orc, run, 0.1, label="after append")


def test_rate_one_equals_plain_decode(orc):
    run = _run(CASES["mix4"])
    q = run.batch.q
    full = H.gpu_decode(run, q).float()
    out, _, sel = H.gpu_decode_select(run, q, 1.0)
    assert float((out.float() - full).abs().max()) <= H.TOL_OUT
    # every candidate slot is kept
    desc = run.cc.desc.cpu().numpy().view(np.uint64)
    S = run.wl.segment_len
    for u in range(desc.shape[0]):
        nsg = int(run.cc.n_segs[u])
        strat = ((desc[u, :nsg] >> np.uint64(32)) & np.uint64(255)).astype(int)
        ncand = sum(run.wl.r if s in (B.TOK, B.BOTH) else S for s in strat)
        assert int(sel[u, :nsg * S].sum()) == ncand


def test_select_batch16_128k_sampled_units(orc):
    wl = synth.WORKLOADS["llama3_8b_b16_128k_mix"]
    batch = synth.generate(wl, seed=0, device="cuda", extra_capacity=16)
    run = H.make_run(wl, batch, H.params_for(wl))
    H.compress(run)
    check_select(orc, run, 0.0625, units=[(0, 0), (7, 3), (15, 7)], label=wl.name)
