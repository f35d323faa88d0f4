"""The three large workloads at their full sizes, in the launch configuration
of the library's normal entry points, on sampled units:

* batch 16 x 128K tokens, budget 15 %, the four-class segment mix, then 256
  decode steps with kv2d_append;
* batch 1 x 1M tokens, S = W = 128, budget 10 %, 0.1 % planted tokens;
* a ragged batch of 32 sequences in [4K, 128K] on 16-token pages, 512 decode
  steps with a re-compression of the trailing region every 128 steps.

For a sampled unit, every compressed byte is checked against the oracle fed
with the GPU's fp32 a_d and s_t (selection, packing and g_t are bit-exact),
decode outputs against the oracle's decode over the same arena, and the
scores themselves either fully (oracle scoring of the whole unit, 128K) or,
at 1M, on window rows the oracle scores one at a time plus the identity
sum_t s_t = G * W that holds at any size.
"""
import numpy as np
import pytest
import torch

from kv_cache_compression_kv2d_b200 import binding as B
from kv_cache_compression_kv2d_b200 import synth

from tests import gpu_harness as H

pytestmark = pytest.mark.gpu


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


def _decode_matches(orc, run, q, units):
    out = H.gpu_decode(run, q).float().cpu().numpy()
    G = run.wl.group
    for b, h in units:
        ref = H.oracle_decode_unit(orc, run, b, h, q)
        err = float(np.max(np.abs(out[b, h * G:(h + 1) * G] - ref)))
        assert err <= H.TOL_OUT, f"decode unit ({b}, {h}): max abs error {err}"


def test_batch16_128k_mix_then_256_decode_steps(orc):
    wl = synth.WORKLOADS["llama3_8b_b16_128k_mix"]
    run = _device_run(wl, wl.decode_steps + 16)
    H.compress(run)
    sampled = [(0, 0), (wl.batch - 1, wl.num_kv_heads - 1)]
    H.check_compress_unit(orc, run, *sampled[0], independent=True)
    H.check_compress_unit(orc, run, *sampled[1], independent=False)
    # every strategy is chosen somewhere in the batch
    desc = run.cc.desc.cpu().numpy().view(np.uint64)
    nsg = run.cc.n_segs.cpu().numpy()
    seen = set()
    for u in range(desc.shape[0]):
        seen |= set(((desc[u, :nsg[u]] >> np.uint64(32)) & np.uint64(255)).astype(int).tolist())
    assert seen == {0, 1, 2, 3}, f"strategies seen: {sorted(seen)}"
    ws = B.workspace(256)
    for step in range(wl.decode_steps):
        k, v, q = synth.decode_tokens(wl, step, device="cuda", mu=run.batch.mu)
        B.kv2d_append(run.p, wl.batch, run.dv, k, v, run.seq_len, ws)
        if step in (0, wl.decode_steps - 1):
            torch.cuda.synchronize()
            _decode_matches(orc, run, q, sampled)
    assert B.kv2d_read_status(ws) == 0


def test_1m_tokens_sampled_rows_and_units(orc):
    wl = synth.WORKLOADS["llama3_8b_1m"]
    run = _device_run(wl, 16)
    H.compress(run)
    b, h = 0, 3
    H.check_compress_unit(orc, run, b, h, independent=False)
    u = b * wl.num_kv_heads + h
    po = H.oracle_params(orc, run.p)
    T = run.dbg["seq_host"][b]
    G, W, d = wl.group, wl.window, wl.head_dim
    # a_d against the oracle
    qw16 = H.unit_qw(run, b, h)
    a_ref = orc.win_stats(po, qw16.astype(np.float64))
    a_gpu = run.dbg["a"][u].double().cpu().numpy()
    assert np.max(np.abs(a_gpu - a_ref) / np.maximum(np.abs(a_ref), 1e-30)) < 1e-5
    # lse of sampled window rows, each scored alone by the oracle: row i of
    # head g sees keys [0, T - W + i], the same set as inside the window
    K16, _ = H.unit_inputs(run, b, h, 0, T)
    Kd = K16.astype(np.float64)
    lse_gpu = run.dbg["lse"][b, h * G:(h + 1) * G].double().cpu().numpy()   # [G][W], natural log
    po1 = orc.params(d, 1, wl.segment_len, 1, wl.r, wl.c, float(np.float32(wl.budget)),
                     float(np.float32(run.p.scale)))
    for g, i in [(0, 0), (1, W // 2), (G - 1, W - 1)]:
        p_i = T - W + i
        lse_ref, _ = orc.score(po1, p_i + 1, 0, Kd[:p_i + 1], qw16[g * W + i:g * W + i + 1].astype(np.float64))
        got = lse_gpu[g, i]
        assert abs(got - lse_ref[0]) / max(1.0, abs(lse_ref[0])) < H.TOL_REL, (g, i, got, lse_ref[0])
    # every row's softmax sums to one, so the token masses sum to G * W (the
    # whole prompt is segments here: no dense tail takes part of the mass)
    n = T - run.dbg["ce_before"][b]
    assert n % wl.segment_len == 0
    s_gpu = run.dbg["s"][u, :n].double().cpu().numpy()
    assert abs(s_gpu.sum() - G * W) <= G * W * H.TOL_REL
    assert np.all(s_gpu >= 0)
    _, _, q = synth.decode_tokens(wl, 0, device="cuda", mu=run.batch.mu)
    _decode_matches(orc, run, q, [(b, h)])


def test_ragged32_paged_periodic_recompression(orc):
    wl = synth.WORKLOADS["ragged32_paged"]
    run = _device_run(wl, wl.decode_steps + 16)
    H.compress(run)
    lens = run.batch.seq_len.tolist()
    b_short, b_long = int(np.argmin(lens)), int(np.argmax(lens))
    sampled = [(b_short, 0), (b_long, wl.num_kv_heads - 1)]
    H.check_compress_unit(orc, run, *sampled[0], independent=True)
    H.check_compress_unit(orc, run, *sampled[1], independent=False)
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
            for bh in sampled:
                H.check_compress_unit(orc, run, *bh, independent=False)
            _decode_matches(orc, run, q, sampled)
    assert events == wl.decode_steps // wl.recompress_every
    assert B.kv2d_read_status(ws) == 0
    assert all(ce > 0 for ce in run.dbg["ce_before"])
