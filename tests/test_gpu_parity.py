"""CUDA path vs the fp64 CPU oracle, element by element, through the C ABI.

Sizes are chosen so that the oracle finishes in seconds while the kernels
still see several tiles, ragged tails, padded window rows (G*W not a multiple
of 128), both pass-2 column modes (G*W <= 256 and > 256), paged and
contiguous dense views, and a region that starts after earlier compressions.
"""
import math

import numpy as np
import pytest
import torch

from kv_cache_compression_kv2d_b200 import binding as B
from kv_cache_compression_kv2d_b200 import synth
from kv_cache_compression_kv2d_b200.synth import Workload

from tests import gpu_harness as H

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": synth.WORKLOADS["tiny"],
    "ragged_multi": Workload("ragged_multi", 3, 2, 4, 128, 1537, 64, 24, 0.3, ragged_min=700),
    "paged": Workload("paged", 3, 2, 4, 128, 1400, 64, 32, 0.25, ragged_min=600, block_size=16),
    "gw512_s128": Workload("gw512_s128", 1, 2, 4, 128, 2048 + 77, 128, 128, 0.15),
    "g8_gw384": Workload("g8_gw384", 2, 1, 8, 128, 1100, 32, 48, 0.3),
    "g2_small_rc": Workload("g2_small_rc", 2, 2, 2, 128, 999, 16, 64, 0.35, keep_tokens=3,
                            keep_channels=20),
    "mix4": Workload("mix4", 2, 2, 4, 128, 2048, 64, 64, 0.15, segment_mix=True),
}


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from kv_cache_compression_kv2d_b200 import build
    build.build()
    assert torch.cuda.is_available()
    B.lib()


def _run(wl, seed=0, budget=None, extra=0, **kw):
    batch = synth.generate(wl, seed=seed, device="cpu", extra_capacity=extra)
    dev = H.to_device(batch)
    p = H.params_for(wl, budget=budget, **kw)
    run = H.make_run(wl, dev, p)
    return run


def _check_all_units(orc, run, independent=True):
    strats = []
    for b in range(run.wl.batch):
        for h in range(run.wl.num_kv_heads):
            res = H.check_compress_unit(orc, run, b, h, independent=independent)
            if res is not None:
                strats.extend(res["strat"].tolist())
    return strats


def _check_decode(orc, run, q=None):
    q = run.batch.q if q is None else q
    out = H.gpu_decode(run, q).float().cpu().numpy()
    worst = 0.0
    for b in range(run.wl.batch):
        for h in range(run.wl.num_kv_heads):
            ref = H.oracle_decode_unit(orc, run, b, h, q)
            G = run.wl.group
            got = out[b, h * G:(h + 1) * G]
            worst = max(worst, float(np.max(np.abs(got - ref))))
    assert worst <= H.TOL_OUT, f"decode max abs err {worst}"
    return worst


@pytest.mark.parametrize("name", list(CASES))
def test_compress_and_decode_parity(orc, name):
    wl = CASES[name]
    run = _run(wl)
    H.compress(run)
    strats = _check_all_units(orc, run)
    assert len(strats) > 0
    _check_decode(orc, run)


def test_mix4_spans_all_strategies(orc):
    run = _run(CASES["mix4"])
    H.compress(run)
    strats = _check_all_units(orc, run, independent=False)
    assert set(strats) == {0, 1, 2, 3}, f"strategies seen: {sorted(set(strats))}"


def test_decode_on_oracle_arena(orc):
    """Decode fed with the oracle's own packed arena (independent scoring),
    uploaded into a fresh compressed cache."""
    wl = CASES["ragged_multi"]
    run = _run(wl, seed=3)
    p = run.p
    po = H.oracle_params(orc, p)
    cc = B.CompressedCache(p, wl.batch, run.batch.capacity)
    S = wl.segment_len
    for b in range(wl.batch):
        T = int(run.batch.seq_len[b])
        nseg = T // S
        for h in range(wl.num_kv_heads):
            u = b * wl.num_kv_heads + h
            K16, V16 = H.unit_inputs(run, b, h, 0, T)
            ref = orc.compress_unit(po, T, 0, K16, V16, H.unit_qw(run, b, h))
            assert ref["status"] == 0
            base = u * cc.arena_stride
            cc.arena[base:base + ref["used"]] = torch.from_numpy(ref["arena"]).cuda()
            d = (ref["offs"] // 16).astype(np.uint64) | (ref["strat"].astype(np.uint64) << np.uint64(32))
            cc.desc[u, :nseg] = torch.from_numpy(d.view(np.int64)).cuda()
            cc.n_segs[u] = nseg
            cc.used_bytes[u] = ref["used"]
        cc.comp_end[b] = nseg * S
    q = run.batch.q
    out = H.gpu_decode(run, q, cc=cc).float().cpu().numpy()
    for b in range(wl.batch):
        for h in range(wl.num_kv_heads):
            ref = H.oracle_decode_unit(orc, run, b, h, q, cc=cc)
            G = wl.group
            assert np.max(np.abs(out[b, h * G:(h + 1) * G] - ref)) <= H.TOL_OUT


def test_full_budget_equals_dense_attention(orc):
    wl = CASES["tiny"].with_(budget=1.0)
    run = _run(wl, budget=1.0)
    H.compress(run)
    strats = _check_all_units(orc, run, independent=False)
    assert set(strats) == {0}
    q = run.batch.q
    out = H.gpu_decode(run, q).float()
    T = int(run.batch.seq_len[0])
    K = run.batch.k[0, :, :T].float()
    V = run.batch.v[0, :, :T].float()
    G = wl.group
    ref = torch.nn.functional.scaled_dot_product_attention(
        q[0].float().view(wl.num_kv_heads, G, 1, wl.head_dim),
        K[:, None], V[:, None], scale=float(run.p.scale)).view(wl.num_q_heads, wl.head_dim)
    assert float((out[0] - ref).abs().max()) <= H.TOL_OUT


def test_subnormal_channel_products(orc):
    """K scaled by 2^-13 (exact in fp16 down to its subnormal grid): the
    channel products |k_x| a_x then lie on both sides of the smallest normal
    fp16, so channel selection ranks fp16 subnormal keys too."""
    wl = CASES["ragged_multi"]
    run = _run(wl, seed=7)
    run.batch.k.mul_(2.0 ** -13)
    H.compress(run)
    strats = _check_all_units(orc, run)
    assert len(strats) > 0
    _check_decode(orc, run)


def test_keep_all_channels_is_token_only(orc):
    wl = CASES["ragged_multi"]
    run = _run(wl, keep_channels=128)
    H.compress(run)
    strats = _check_all_units(orc, run, independent=False)
    assert set(strats) <= {0, 1}
    _check_decode(orc, run)


def test_append_then_periodic_compress(orc):
    """Decode steps append tokens; a second compression covers the trailing
    region [comp_end, seq_len) only, appending to the same arenas."""
    wl = CASES["paged"]
    steps = 150
    run = _run(wl, extra=steps + 16)
    H.compress(run)
    _check_all_units(orc, run)
    ws = B.workspace(256)
    for step in range(steps):
        k, v, q = synth.decode_tokens(wl, step, device="cuda", mu=run.batch.mu)
        B.kv2d_append(run.p, wl.batch, run.dv, k, v, run.seq_len, ws)
        if step in (0, steps - 1):
            torch.cuda.synchronize()
            _check_decode(orc, run, q)
    torch.cuda.synchronize()
    assert B.kv2d_read_status(ws) == 0
    seq = run.seq_len.cpu().tolist()
    assert seq == [int(x) + steps for x in run.batch.seq_len.tolist()]
    # appended rows landed in the dense view
    k, v, _ = synth.decode_tokens(wl, steps - 1, device="cuda", mu=run.batch.mu)
    for b in range(wl.batch):
        kr, vr = synth.dense_rows(run.batch, b, 1, seq[b] - 1, seq[b])
        assert torch.equal(kr[0], k[b, 1]) and torch.equal(vr[0], v[b, 1])
    # the window queries of the second compression: fresh draws
    g = torch.Generator(device="cuda")
    g.manual_seed(99)
    run.batch.qw = (run.batch.mu.repeat_interleave(wl.group, 0)[None, :, None, :] +
                    torch.randn(run.batch.qw.shape, generator=g, device="cuda")).to(torch.float16)
    H.compress(run, seq_host=seq)
    assert any(ce > 0 for ce in run.dbg["ce_before"])
    _check_all_units(orc, run)
    _, _, q = synth.decode_tokens(wl, steps, device="cuda", mu=run.batch.mu)
    _check_decode(orc, run, q)


def test_decode_is_deterministic(orc):
    run = _run(CASES["mix4"])
    H.compress(run)
    q = run.batch.q
    a = H.gpu_decode(run, q)
    b = H.gpu_decode(run, q)
    assert torch.equal(a, b)


def test_compress_is_deterministic(orc):
    wl = CASES["g8_gw384"]
    r1 = _run(wl, seed=5)
    H.compress(r1)
    r2 = _run(wl, seed=5)
    H.compress(r2)
    assert torch.equal(r1.cc.arena, r2.cc.arena)
    assert torch.equal(r1.cc.desc, r2.cc.desc)
    a, b = r1.dbg["s"], r2.dbg["s"]          # NaN-filled beyond each region
    assert torch.equal(torch.isnan(a), torch.isnan(b))
    assert torch.equal(torch.nan_to_num(a), torch.nan_to_num(b))


def test_llama8b_32k_layer_all_units(orc):
    """Full-size Llama-3-8B-shaped layer (8 KV heads, 32K tokens, budget
    20%): every unit against the oracle, in the launch configuration the
    benchmark times."""
    wl = synth.WORKLOADS["llama3_8b_32k"]
    run = _run(wl)
    H.compress(run)
    from oracle.oracle import parallel_map  # noqa: F401  (threads inside the C oracle)
    units = [(b, h) for b in range(wl.batch) for h in range(wl.num_kv_heads)]
    res = parallel_map(lambda bh: H.check_compress_unit(orc, run, bh[0], bh[1]), units)
    assert all(r is not None for r in res)
    _check_decode(orc, run)


@pytest.mark.parametrize("keep_channels", [32, 20, 48])
def test_channel_ties_parity(orc, keep_channels):
    """Keys rounded to multiples of 0.5 (and a constant row) make many
    channel products tie exactly at the top-c cut: the selection must still
    match the oracle bit for bit (ties to the lower channel)."""
    wl = Workload("ties", 1, 2, 4, 128, 1024, 64, 32, 0.3)
    batch = synth.generate(wl, seed=21)
    batch.k[:] = (batch.k.float() * 2).round().div(2).to(torch.float16)
    batch.k[0, 0, 100] = 1.0
    batch.qw[:] = (batch.qw.float() * 2).round().div(2).to(torch.float16)
    run = H.make_run(wl, H.to_device(batch), H.params_for(wl, keep_channels=keep_channels))
    H.compress(run)
    _check_all_units(orc, run, independent=False)
    _check_decode(orc, run)


@pytest.mark.parametrize("keep_tokens", [3, 4, 8, 16])
def test_token_ties_parity(orc, keep_tokens):
    """Window queries of zero give every visible key the same logit, so the
    token masses of all keys that every window row sees are equal: the top-r
    of each segment is decided by the tie rule alone (lower token first),
    and the zero channel weights make every channel tie as well (lower
    channel first).  Covers both segment-select kernels (r = 3 runs the
    warp-per-segment one, r = 4, 8, 16 the thread-per-segment one)."""
    wl = Workload("token_ties", 2, 1, 4, 128, 1280, 64, 32, 0.3, ragged_min=900)
    batch = synth.generate(wl, seed=4)
    batch.qw.zero_()
    run = H.make_run(wl, H.to_device(batch), H.params_for(wl, keep_tokens=keep_tokens))
    H.compress(run)
    _check_all_units(orc, run, independent=True)
    _check_decode(orc, run)


@pytest.mark.parametrize("name,gamma,alpha", [("tiny", 8, 4), ("mix4", 6, 3), ("g2_small_rc", 4, 1),
                                               ("gw512_s128", 8, 8), ("paged", 5, 2)])
def test_token2chunk_parity(orc, name, gamma, alpha):
    """Kara's Token2Chunk variant of the kept tokens (core top r - alpha,
    gaps of span <= gamma filled by summed mass within the budget alpha,
    the rest from the best tokens left): the whole compression against the
    oracle -- scores independently, and with the GPU's scores fed in the
    kept tokens, strategies and every packed byte bit for bit -- then
    decode."""
    wl = CASES[name]
    run = _run(wl, chunk_len=gamma, chunk_budget=alpha)
    H.compress(run)
    strats = _check_all_units(orc, run, independent=True)
    assert len(strats) > 0
    _check_decode(orc, run)


@pytest.mark.parametrize("cap", [32, 41])
def test_decode_block_table_in_chunks(orc, cap):
    """With more units than half the SMs the batch's bytes are shared out
    over the CTAs, and each CTA tables its blocks in chunks of whole
    segments; a cap of 32 or 41 blocks per chunk makes every share take
    several chunks (a 64-token segment is 8 blocks, so 41 leaves a remainder),
    with the dense tail after the last chunk."""
    wl = Workload("chunks", 40, 2, 4, 128, 1601, 64, 64, 0.15, ragged_min=900, segment_mix=True)
    run = _run(wl, seed=5)
    H.compress(run)
    B.kv2d_set_decode_table_cap(cap)
    try:
        _check_decode(orc, run)
    finally:
        B.kv2d_set_decode_table_cap(0)


def test_decode_in_cuda_graph(orc):
    """kv2d_decode_attn is capturable in a CUDA graph (no host sync, fixed
    grid from the host maxima, tickets back at zero after every call): three
    captured calls replayed give the direct call's output bit for bit."""
    wl = CASES["ragged_multi"]
    run = _run(wl, seed=2)
    H.compress(run)
    q = run.batch.q
    ref = H.gpu_decode(run, q)
    p = run.p
    ws = B.workspace(B.kv2d_workspace_bytes(p, B.OP_DECODE, wl.batch, run.batch.capacity))
    out = torch.full_like(ref, float("nan"))
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=s):
        for _ in range(3):
            B.kv2d_decode_attn(p, wl.batch, run.cc.struct, run.dv, run.seq_len, run.batch.capacity,
                               q, out, ws, stream=s)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(2):
        out.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        assert torch.equal(out, ref)
    assert B.kv2d_read_status(ws) == 0


def _tail_only_decode(lengths, group=4, hkv=2, d=128):
    """Decode over dense tails only (nothing compressed): sequence b holds
    lengths[b] tokens.  Returns (out, k, v, q) on the device."""
    batch = len(lengths)
    cap = 300   # > 256: two CTAs per unit allowed, so 80 units ask for all 148
    g = torch.Generator(device="cuda").manual_seed(17)
    k = torch.randn((batch, hkv, cap, d), generator=g, device="cuda").to(torch.float16)
    v = torch.randn((batch, hkv, cap, d), generator=g, device="cuda").to(torch.float16)
    q = torch.randn((batch, hkv * group, d), generator=g, device="cuda").to(torch.float16)
    p = B.params(d, hkv * group, hkv, 64, 32, 8, 32, 0.25, float(np.float32(1.0 / np.sqrt(d))))
    cc = B.CompressedCache(p, batch, cap)
    seq = torch.tensor(lengths, dtype=torch.int32, device="cuda")
    out = torch.full((batch, hkv * group, d), float("nan"), dtype=torch.float16, device="cuda")
    ws = B.workspace(B.kv2d_workspace_bytes(p, B.OP_DECODE, batch, cap))
    B.kv2d_decode_attn(p, batch, cc.struct, B.dense(k, v), seq, cap, q, out, ws)
    torch.cuda.synchronize()
    assert B.kv2d_read_status(ws) == 0
    return out, k, v, q


def test_decode_empty_batch_leaves_ctas_without_bytes(orc):
    """80 units with no token at all: the batch-wide range holds 80 bytes
    (one per unit) for 148 CTAs, so most CTAs get an empty share; each unit
    still gets exactly one writer, and a unit without tokens decodes to 0."""
    out, _, _, _ = _tail_only_decode([0] * 40)
    assert torch.equal(out, torch.zeros_like(out))


def test_decode_one_token_over_many_empty_pieces(orc):
    """One sequence with a single dense token among 39 empty ones: its two
    units span ~70 CTAs each, all but one with no token, and the merge of
    those pieces must give that token's value row exactly (softmax weight 1)."""
    lengths = [0] * 39 + [1]
    out, _, v, _ = _tail_only_decode(lengths)
    G = 4
    for b in range(40):
        for h in range(2):
            got = out[b, h * G:(h + 1) * G]
            if lengths[b] == 0:
                assert torch.equal(got, torch.zeros_like(got))
            else:
                assert torch.equal(got, v[b, h, 0].expand(G, -1))
