"""Pins of the oracle's decode-time token selection (stage 2) against facts
that do not come from its own arithmetic: a rate that keeps every candidate
reduces to the full decode (itself pinned to textbook attention); scores
against the test's own byte parser and a numpy dot product; the selection
against a stable sort by (score desc, slot asc); the attention against an
independent masked evaluation through the library softmax; the count in
closed form; hand-built ties; weights that sum to one.
"""
import math

import numpy as np
import torch

from tests.test_oracle_pins import BOTH, CH, FULL, TOK, _parse, _textbook, _unit, f16


def _compressed(orc, seed, S=16, d=32, G=4, W=8, r=3, c=7, beta=0.3, nseg=9, tail=5):
    p = orc.params(d, G, S, W, r, c, beta)
    rng = np.random.default_rng(seed)
    T = S * nseg + tail
    K16, V16, qw16, q16 = _unit(rng, S, d, G, T, W)
    res = orc.compress_unit(p, T, 0, K16, V16, qw16)
    assert res["status"] == 0
    return p, res, K16, V16, q16


def _candidates(orc, p, res):
    """Kept keys and values of every candidate slot j*S + i, from the
    test's own parser (dropped channels zero)."""
    S, d = p.S, p.d
    keys, vals, slots = [], [], []
    for j in range(res["nseg"]):
        st = int(res["strat"][j])
        end = res["offs"][j + 1] if j + 1 < res["nseg"] else res["used"]
        t_, K_, ci_, kv_, V_ = _parse(p, orc, st, res["arena"][res["offs"][j]:end])
        n = V_.shape[0]
        if K_ is not None:
            Kd = K_.view(np.float16).astype(np.float64)
        else:
            Kd = np.zeros((n, d))
            for t in range(n):
                Kd[t, ci_[t].astype(np.int64)] = kv_[t].view(np.float16).astype(np.float64)
        for i in range(n):
            keys.append(Kd[i])
            vals.append(V_[i].view(np.float16).astype(np.float64))
            slots.append(j * S + i)
    return np.array(keys), np.array(vals), np.array(slots)


def test_scores_are_max_over_heads_of_kept_key_logits(orc):
    p, res, _, _, q16 = _compressed(orc, 31)
    assert len(set(res["strat"].tolist())) >= 2
    score, ncand = orc.select_scores(p, res["arena"], res["offs"], res["strat"], q16)
    keys, _, slots = _candidates(orc, p, res)
    assert ncand == len(slots)
    want = np.full(res["nseg"] * p.S, -np.inf)
    want[slots] = (p.scale * (q16.astype(np.float64) @ keys.T)).max(axis=0)
    assert np.array_equal(np.isinf(score), np.isinf(want))
    fin = np.isfinite(want)
    assert np.max(np.abs(score[fin] - want[fin])) < 1e-12


def test_scores_over_every_strategy(orc):
    """Segments packed as FULL, CH, TOK, BOTH, CH, BOTH (the oracle's own
    packer, its selection steps not involved): every candidate's score is
    the max over heads of the logit of its key as the test's parser reads
    it, dropped channels zero."""
    S, d, G, r, c = 8, 32, 4, 3, 5
    p = orc.params(d, G, S, 8, r, c, 0.3)
    rng = np.random.default_rng(57)
    strat = np.array([FULL, CH, TOK, BOTH, CH, BOTH], np.int32)
    nseg = len(strat)
    K16 = f16(rng.standard_normal((nseg * S, d)))
    V16 = f16(rng.standard_normal((nseg * S, d)))
    q16 = f16(rng.standard_normal((G, d)))
    arena, offs, o = [], [], 0
    for j in range(nseg):
        tidx = np.sort(rng.choice(S, r, replace=False)).astype(np.uint8)
        cidx_all = np.stack([np.sort(rng.choice(d, c, replace=False)) for _ in range(S)]).astype(np.uint8)
        buf = orc.pack_segment(p, strat[j], K16[j * S:(j + 1) * S], V16[j * S:(j + 1) * S], tidx, cidx_all)
        offs.append(o)
        arena.append(buf)
        o += buf.size
    res = {"nseg": nseg, "strat": strat, "arena": np.concatenate(arena), "offs": np.array(offs),
           "used": o}
    score, ncand = orc.select_scores(p, res["arena"], res["offs"], res["strat"], q16)
    keys, _, slots = _candidates(orc, p, res)
    assert ncand == len(slots) == 3 * S + 3 * r   # FULL, CH, CH keep S; TOK, BOTH, BOTH keep r
    want = np.full(nseg * S, -np.inf)
    want[slots] = (p.scale * (q16.astype(np.float64) @ keys.T)).max(axis=0)
    assert np.array_equal(np.isinf(score), np.isinf(want))
    fin = np.isfinite(want)
    assert np.max(np.abs(score[fin] - want[fin])) < 1e-12


def test_selection_is_a_stable_sort_by_score(orc):
    rng = np.random.default_rng(32)
    score = rng.standard_normal(200)
    score[rng.choice(200, 40, replace=False)] = -np.inf
    score[[10, 50, 51, 120]] = 0.5          # exact ties: the lower slots win
    for n_sel in (0, 1, 3, 17, 160, 200):
        sel = orc.select_tokens(score, n_sel)
        fin = np.flatnonzero(np.isfinite(score))
        order = fin[np.lexsort((fin, -score[fin]))]
        want = np.zeros(200, np.uint8)
        want[order[:n_sel]] = 1
        assert np.array_equal(sel, want), n_sel
    # two of three tied maxima
    s = np.array([1.0, 2.0, 2.0, -np.inf, 2.0])
    assert orc.select_tokens(s, 2).tolist() == [0, 1, 1, 0, 0]


def test_count_in_closed_form(orc):
    p = orc.params(128, 4, 64, 64, 8, 32, 0.2)
    assert orc.select_count(p, 2, 100, 0.0625) == 8          # ceil(0.0625 * 128)
    assert orc.select_count(p, 2, 100, 0.0626) == 9          # ceil(8.0128)
    assert orc.select_count(p, 2, 5, 0.0625) == 5            # capped by the candidates
    assert orc.select_count(p, 2, 100, 1.0) == 100
    assert orc.select_count(p, 3, 40, 0.125) == 24
    assert orc.select_count(p, 0, 0, 0.5) == 0


def test_all_candidates_reduce_to_full_decode(orc):
    p, res, K16, V16, q16 = _compressed(orc, 33)
    nc = res["nseg"] * p.S
    score, ncand = orc.select_scores(p, res["arena"], res["offs"], res["strat"], q16)
    n = orc.select_count(p, res["nseg"], ncand, 1.0)
    sel = orc.select_tokens(score, n)
    assert int(sel.sum()) == ncand
    out = orc.decode_select(p, res["arena"], res["offs"], res["strat"], sel, K16[nc:], V16[nc:], q16)
    full = orc.decode_unit(p, res["arena"], res["offs"], res["strat"], K16[nc:], V16[nc:], q16)
    assert np.max(np.abs(out - full)) < 1e-12


def test_selected_attention_matches_independent_masked_softmax(orc):
    for seed, rho in ((34, 0.0625), (35, 0.125), (36, 0.3)):
        p, res, K16, V16, q16 = _compressed(orc, seed, beta=0.5)
        nc = res["nseg"] * p.S
        score, ncand = orc.select_scores(p, res["arena"], res["offs"], res["strat"], q16)
        n = orc.select_count(p, res["nseg"], ncand, rho)
        assert n == min(ncand, math.ceil(rho * nc))
        sel = orc.select_tokens(score, n)
        keys, vals, slots = _candidates(orc, p, res)
        keep = sel[slots].astype(bool)
        assert int(keep.sum()) == n
        K = np.concatenate([keys[keep], K16[nc:].astype(np.float64)])
        V = np.concatenate([vals[keep], V16[nc:].astype(np.float64)])
        ref = _textbook(q16.astype(np.float64), K, V, p.scale)
        out = orc.decode_select(p, res["arena"], res["offs"], res["strat"], sel, K16[nc:],
                                V16[nc:], q16)
        assert np.max(np.abs(out - ref)) < 1e-12


def test_selected_weights_sum_to_one(orc):
    p, res, K16, _, q16 = _compressed(orc, 37)
    T = K16.shape[0]
    V16 = f16(np.full((T, p.d), 1.5))
    res = orc.compress_unit(p, T, 0, K16, V16, np.zeros((p.G * p.W, p.d), np.float16))
    nc = res["nseg"] * p.S
    score, ncand = orc.select_scores(p, res["arena"], res["offs"], res["strat"], q16)
    sel = orc.select_tokens(score, orc.select_count(p, res["nseg"], ncand, 0.1))
    out = orc.decode_select(p, res["arena"], res["offs"], res["strat"], sel, K16[nc:], V16[nc:], q16)
    assert np.max(np.abs(out - 1.5)) < 1e-12


def test_no_tokens_at_all_gives_zero(orc):
    p = orc.params(32, 2, 16, 4, 3, 7, 0.3)
    q16 = f16(np.ones((2, 32)))
    out = orc.decode_select(p, np.zeros(0, np.uint8), np.zeros(0, np.int64), np.zeros(0, np.int32),
                            np.zeros(0, np.uint8), np.zeros((0, 32), np.float16),
                            np.zeros((0, 32), np.float16), q16)
    assert not out.any()
