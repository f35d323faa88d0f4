"""The three large workloads at their full sizes, in the launch configuration
of the library's normal entry points, on sampled units (four per workload):

* batch 16 x 128K tokens, budget 15 %, the four-class segment mix, then 256
  decode steps with kv2d_append;
* batch 1 x 1M tokens, S = W = 128 (G * W = 512: pass 2 in split-column
  mode), budget 10 %, 0.1 % planted tokens;
* a ragged batch of 32 sequences in [4K, 128K] on 16-token pages, 512 decode
  steps with a re-compression of the trailing region every 128 steps.

For every sampled unit, every compressed byte is checked against the oracle
fed with the GPU's fp32 a_d and s_t (selection, packing and g_t are
bit-exact), and decode outputs against the oracle's decode over the same
arena.  For two units per workload the scores themselves are compared
element by element with the oracle's own (every key of the unit, the 1M one
included: the oracle scores each query head on its own host thread), and
the fully independent end-to-end oracle (its own scores, selection, packing
and decode) is run beside the GPU: the share of segments on which both pick
the same strategy and the decode difference are printed and bounded.
"""
import numpy as np
import pytest
import torch

from kv_cache_compression_kv2d_b200 import binding as B
from kv_cache_compression_kv2d_b200 import synth

from tests import gpu_harness as H

pytestmark = pytest.mark.gpu

# the independent end-to-end oracle takes its own decisions on its own fp64
# scores; near-ties may go the other way, so the whole-pipeline comparison
# is bounded looser than the fed-mode one
MIN_AGREEMENT = 0.98
TOL_END_TO_END = 1e-2


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from kv_cache_compression_kv2d_b200 import build
    build.build()
    assert torch.cuda.is_available()
    B.lib()


def _device_run(wl, extra):
    batch = synth.generate(wl, seed=0, device="cuda", extra_capacity=extra)
    run = H.make_run(wl, batch, H.params_for(wl))
    return run


def _decode_matches(orc, run, q, units, out=None):
    out = H.gpu_decode(run, q).float().cpu().numpy() if out is None else out
    G = run.wl.group
    for b, h in units:
        ref = H.oracle_decode_unit(orc, run, b, h, q)
        err = float(np.max(np.abs(out[b, h * G:(h + 1) * G] - ref)))
        assert err <= H.TOL_OUT, f"decode unit ({b}, {h}): max abs error {err}"
    return out


def _independent(orc, run, units):
    """Scores of each unit against the oracle's own, element by element."""
    scores = {}
    for b, h in units:
        scores[(b, h)] = H.oracle_scores(orc, run, b, h)
        H.check_scores(run, b, h, scores[(b, h)])
    return scores


def _end_to_end(orc, run, scores, q, label):
    """Protocol item 4: the fully independent oracle beside the GPU."""
    out = H.gpu_decode(run, q).float().cpu().numpy()
    G = run.wl.group
    agree = total = 0
    worst = 0.0
    for (b, h), sc in scores.items():
        (a, n), o_ref = H.end_to_end_unit(orc, run, b, h, sc, q)
        agree += a
        total += n
        worst = max(worst, float(np.max(np.abs(out[b, h * G:(h + 1) * G] - o_ref))))
    frac = agree / max(total, 1)
    print(f"\nEND-TO-END {label}: strategy agreement {agree}/{total} = {frac:.4f}, "
          f"decode max abs difference {worst:.3e}")
    assert frac >= MIN_AGREEMENT, f"strategy agreement {frac}"
    assert worst <= TOL_END_TO_END, f"end-to-end decode difference {worst}"


def _strategies_seen(run):
    desc = run.cc.desc.cpu().numpy().view(np.uint64)
    nsg = run.cc.n_segs.cpu().numpy()
    seen = set()
    for u in range(desc.shape[0]):
        seen |= set(((desc[u, :nsg[u]] >> np.uint64(32)) & np.uint64(255)).astype(int).tolist())
    return seen


def test_batch16_128k_mix_then_256_decode_steps(orc):
    wl = synth.WORKLOADS["llama3_8b_b16_128k_mix"]
    run = _device_run(wl, wl.decode_steps + 16)
    H.compress(run)
    sampled = [(0, 0), (5, 3), (10, 6), (wl.batch - 1, wl.num_kv_heads - 1)]
    scores = _independent(orc, run, [sampled[0], sampled[2]])
    for bh in sampled:
        H.check_compress_unit(orc, run, *bh, independent=False)
    assert _strategies_seen(run) == {0, 1, 2, 3}
    _, _, q0 = synth.decode_tokens(wl, 0, device="cuda", mu=run.batch.mu)
    _end_to_end(orc, run, scores, q0, wl.name)
    ws = B.workspace(256)
    for step in range(wl.decode_steps):
        k, v, q = synth.decode_tokens(wl, step, device="cuda", mu=run.batch.mu)
        B.kv2d_append(run.p, wl.batch, run.dv, k, v, run.seq_len, ws)
        if step in (0, wl.decode_steps - 1):
            torch.cuda.synchronize()
            _decode_matches(orc, run, q, sampled)
    assert B.kv2d_read_status(ws) == 0


def test_1m_tokens_sampled_units(orc):
    wl = synth.WORKLOADS["llama3_8b_1m"]
    run = _device_run(wl, 16)
    H.compress(run)
    sampled = [(0, 0), (0, 3), (0, 5), (0, 7)]
    # every key of two units against the oracle: 4 heads x 128 rows x 1M keys
    scores = _independent(orc, run, [sampled[0], sampled[2]])
    for bh in sampled:
        H.check_compress_unit(orc, run, *bh, independent=False)
    # the whole prompt is segments (no dense tail), so every row's softmax
    # mass lands on them: sum_t s_t = G * W for every unit of the batch
    G, W = wl.group, wl.window
    n = run.dbg["seq_host"][0] - run.dbg["ce_before"][0]
    assert n % wl.segment_len == 0
    s_all = run.dbg["s"][:, :n].double()
    sums = s_all.sum(dim=1).cpu().numpy()
    assert np.all(np.abs(sums - G * W) <= G * W * H.TOL_REL), sums
    assert bool((s_all >= 0).all())
    _, _, q = synth.decode_tokens(wl, 0, device="cuda", mu=run.batch.mu)
    out = _decode_matches(orc, run, q, sampled)
    del out
    _end_to_end(orc, run, scores, q, wl.name)


def test_ragged32_paged_periodic_recompression(orc):
    wl = synth.WORKLOADS["ragged32_paged"]
    run = _device_run(wl, wl.decode_steps + 16)
    H.compress(run)
    lens = run.batch.seq_len.tolist()
    order = np.argsort(lens, kind="stable")
    b_short, b_mid, b_long = int(order[0]), int(order[len(order) // 2]), int(order[-1])
    b_q = int(order[len(order) // 4])
    sampled = [(b_short, 0), (b_q, 2), (b_mid, 5), (b_long, wl.num_kv_heads - 1)]
    scores = _independent(orc, run, [sampled[0], sampled[2]])
    for bh in sampled:
        H.check_compress_unit(orc, run, *bh, independent=False)
    _, _, q0 = synth.decode_tokens(wl, 0, device="cuda", mu=run.batch.mu)
    _end_to_end(orc, run, scores, q0, wl.name)
    ws = B.workspace(256)
    events = 0
    for step in range(wl.decode_steps):
        k, v, q = synth.decode_tokens(wl, step, device="cuda", mu=run.batch.mu)
        B.kv2d_append(run.p, wl.batch, run.dv, k, v, run.seq_len, ws)
        if (step + 1) % wl.recompress_every == 0:
            torch.cuda.synchronize()
            seq = run.seq_len.cpu().tolist()
            H.compress(run, seq_host=seq)
            events += 1
            for i, bh in enumerate(sampled):
                # the trailing region is scored again: check its scores fully
                # on two units, the selection and bytes on all four
                H.check_compress_unit(orc, run, *bh, independent=(i % 2 == 0))
            _decode_matches(orc, run, q, sampled)
    assert events == wl.decode_steps // wl.recompress_every
    assert B.kv2d_read_status(ws) == 0
    assert all(ce > 0 for ce in run.dbg["ce_before"])
