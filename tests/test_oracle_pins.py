"""Pins of the fp64 CPU oracle against facts that do not come from the oracle.

Each test names what fixes the expected value: a closed form worked out by
hand, an invariant of the definition, a brute-force enumeration, a library
routine for a special case, or an independent re-implementation of a reading
(the packed-byte parser).  A plausible mistake in the oracle -- a dropped
term, a wrong sign or index, a transposed operand, a wrong tie-break -- fails
at least one of them.
"""
import itertools
import math

import numpy as np
import pytest
import torch

FULL, TOK, CH, BOTH = 0, 1, 2, 3


def f16(x):
    return np.asarray(x, dtype=np.float16)


# ------------------------------------------------------------------ fp16


def test_half_to_double_exhaustive(orc):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    got = np.array([orc.half_to_double(int(b)) for b in bits])
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan], ref[~nan])


# ------------------------------------------------------------- sizes


@pytest.mark.parametrize("S,d,r,c", [(64, 128, 8, 32), (128, 128, 16, 32), (16, 64, 3, 5),
                                     (256, 256, 32, 64), (64, 128, 64, 128)])
def test_segment_bytes_closed_form(orc, S, d, r, c):
    p = orc.params(d, 4, S, 16, r, c, 0.2)
    up = lambda x: -(-x // 16) * 16  # noqa: E731
    assert orc.segment_bytes(p, FULL) == 4 * S * d
    assert orc.segment_bytes(p, TOK) == up(r) + 4 * r * d
    assert orc.segment_bytes(p, CH) == up(S * c) + up(2 * S * c) + 2 * S * d
    assert orc.segment_bytes(p, BOTH) == up(r) + up(r * c) + up(2 * r * c) + 2 * r * d


def test_segment_bytes_default_table(orc):
    # d=128, S=64 (r=8, c=32) and S=128 (r=16, c=32): FULL/TOK/CH/BOTH bytes.
    p = orc.params(128, 4, 64, 64, 8, 32, 0.2)
    assert [orc.segment_bytes(p, k) for k in range(4)] == [32768, 4112, 22528, 2832]
    p = orc.params(128, 4, 128, 128, 16, 32, 0.1)
    assert [orc.segment_bytes(p, k) for k in range(4)] == [65536, 8208, 45056, 5648]


# ---------------------------------------------------------- step 1: a_d


def test_win_stats_closed_form(orc):
    G, W, d = 4, 8, 16
    p = orc.params(d, G, 16, W, 2, 4, 0.2)
    rows = G * W
    qw = np.array([[(-1) ** row * (row + 1) * (k + 1) for k in range(d)] for row in range(rows)],
                  dtype=np.float64)
    a = orc.win_stats(p, qw)
    # mean over rows of (row+1)(k+1) = (k+1)(rows+1)/2
    assert np.array_equal(a, np.array([(k + 1) * (rows + 1) / 2 for k in range(d)]))


# ------------------------------------------------------- steps 2-3: s_t


def test_score_uniform_closed_form(orc):
    """Q = 0: every visible logit is 0, so row i spreads 1 evenly over the
    p_i - r0 + 1 keys it sees (causal, normalised over the region only)."""
    G, W, d, T, r0 = 2, 5, 8, 40, 16
    p = orc.params(d, G, 8, W, 2, 2, 0.2)
    rng = np.random.default_rng(1)
    K = rng.standard_normal((T - r0, d))
    lse, s = orc.score(p, T, r0, K, np.zeros((G * W, d)))
    for g in range(G):
        for i in range(W):
            assert abs(lse[g * W + i] - math.log(T - W + i - r0 + 1)) < 1e-12
    exp = np.zeros(T - r0)
    for t in range(r0, T):
        for i in range(W):
            if t <= T - W + i:
                exp[t - r0] += G / (T - W + i - r0 + 1)
    assert np.max(np.abs(s - exp)) < 1e-12


def test_score_two_key_logistic(orc):
    """One row, two keys: s_0 = 1 / (1 + exp(scale*q.(k1-k0)))."""
    d = 4
    p = orc.params(d, 1, 2, 1, 1, 1, 0.5, scale=0.5)
    q = np.array([[1.0, -2.0, 0.5, 3.0]])
    K = np.array([[0.5, 0.25, -1.0, 2.0], [1.0, 1.0, 0.0, -0.5]])
    lse, s = orc.score(p, 2, 0, K, q)
    l0 = 0.5 * (0.5 - 0.5 - 0.5 + 6.0)
    l1 = 0.5 * (1.0 - 2.0 + 0.0 - 1.5)
    assert abs(s[0] - 1 / (1 + math.exp(l1 - l0))) < 1e-15
    assert abs(s[1] - 1 / (1 + math.exp(l0 - l1))) < 1e-15
    assert abs(lse[0] - math.log(math.exp(l0) + math.exp(l1))) < 1e-14


def test_score_mass_invariant_and_dominant_key(orc):
    G, W, d, T, r0 = 4, 8, 32, 200, 64
    p = orc.params(d, G, 8, W, 2, 2, 0.2)
    rng = np.random.default_rng(2)
    K = rng.standard_normal((T - r0, d))
    mu = rng.standard_normal(d)
    qw = mu[None, :] + 0.1 * rng.standard_normal((G * W, d))
    lse, s = orc.score(p, T, r0, K, qw)
    assert abs(s.sum() - G * W) < 1e-9          # each row's softmax sums to 1
    tstar = 37                                  # visible to every row
    K2 = K.copy()
    K2[tstar] = 400.0 * mu / np.dot(mu, mu)
    _, s2 = orc.score(p, T, r0, K2, qw)
    assert s2[tstar] > G * W * (1 - 1e-6)


def test_score_permutation_equivariance(orc):
    G, W, d, T, r0 = 2, 6, 16, 120, 32
    p = orc.params(d, G, 8, W, 2, 2, 0.2)
    rng = np.random.default_rng(3)
    K = rng.standard_normal((T - r0, d))
    qw = rng.standard_normal((G * W, d))
    lse, s = orc.score(p, T, r0, K, qw)
    n_full = T - W + 1 - r0                     # keys seen by every row
    perm = np.concatenate([rng.permutation(n_full), np.arange(n_full, T - r0)])
    lse2, s2 = orc.score(p, T, r0, K[perm], qw)
    assert np.max(np.abs(lse2 - lse)) < 1e-12
    assert np.max(np.abs(s2 - s[perm])) < 1e-12


def test_score_splits_by_query_head(orc):
    """Each window row's softmax involves only its own query, so scoring the
    G heads as G single-head problems gives the same lse rows, and s_t (a sum
    over rows) is the sum of the heads' shares.  The full-size GPU tests rely
    on this to score a large unit one head per host thread."""
    rng = np.random.default_rng(3)
    G, W, d, T, r0 = 4, 8, 128, 300, 64
    K = f16(rng.standard_normal((T - r0, d))).astype(np.float64)
    qw = f16(rng.standard_normal((G * W, d))).astype(np.float64)
    p = orc.params(d, G, 16, W, 2, 32, 0.5)
    lse, s = orc.score(p, T, r0, K, qw)
    p1 = orc.params(d, 1, 16, W, 2, 32, 0.5)
    s_sum = np.zeros_like(s)
    for g in range(G):
        lse_g, s_g = orc.score(p1, T, r0, K, qw[g * W:(g + 1) * W])
        assert np.array_equal(lse_g, lse[g * W:(g + 1) * W])
        s_sum += s_g
    assert np.allclose(s_sum, s, rtol=1e-12, atol=0)


def test_score_rejects_window_beyond_region(orc):
    p = orc.params(8, 1, 8, 10, 2, 2, 0.2)
    with pytest.raises(ValueError):
        orc.score(p, 20, 12, np.zeros((8, 8)), np.zeros((10, 8)))


# ------------------------------------------------- step 4: channels, g_t


def test_channel_closed_forms(orc):
    d, c = 16, 5
    p = orc.params(d, 1, 4, 1, 1, c, 0.2)
    rng = np.random.default_rng(4)
    rows = []
    for _ in range(6):
        mags = rng.permutation(d) + 1.0
        sign = rng.choice([-1.0, 1.0], d)
        rows.append(mags * sign)
    K = np.array(rows)
    cidx, g = orc.channel(p, K, np.ones(d))
    for t in range(len(rows)):
        mags = np.abs(K[t])
        want = np.sort(np.argsort(-mags)[:c])
        assert np.array_equal(cidx[t], want)
        # dropped magnitudes are 1..d-c: sum (d-c)(d-c+1)/2 over d(d+1)/2
        assert abs(g[t] - (d - c) * (d - c + 1) / (d * (d + 1))) < 1e-15
    # all ties: the lowest c channels, g = (d-c)/d
    cidx, g = orc.channel(p, np.full((2, d), -3.0), np.full(d, 0.5))
    assert np.array_equal(cidx[0], np.arange(c)) and abs(g[0] - (d - c) / d) < 1e-15
    # unit keys: the ranking comes from a alone
    a = rng.permutation(d) + 0.5
    cidx, _ = orc.channel(p, np.ones((1, d)), a)
    assert np.array_equal(cidx[0], np.sort(np.argsort(-a)[:c]))
    # zero row: g = 0 by definition
    _, g = orc.channel(p, np.zeros((1, d)), a)
    assert g[0] == 0.0


def test_channel_against_full_sort(orc):
    d, c = 128, 32
    p = orc.params(d, 1, 4, 1, 1, c, 0.2)
    rng = np.random.default_rng(5)
    K = f16(rng.standard_normal((300, d)) * 2).astype(np.float64)
    K[:, 7] = K[:, 9]                          # planted ties
    K[10:20, :] = np.round(K[10:20, :])        # many ties
    a = f16(rng.random(d) + 0.1).astype(np.float32).astype(np.float64)
    a[9] = a[7]
    cidx, g = orc.channel(p, K, a)
    for t in range(K.shape[0]):
        e = np.abs(K[t]) * a
        order = np.lexsort((np.arange(d), -e))   # e desc, then index asc
        want = np.sort(order[:c])
        assert np.array_equal(cidx[t], want)
        drop = np.setdiff1d(np.arange(d), want)
        assert abs(g[t] - e[drop].sum() / e.sum()) < 1e-13


def test_channel_keep_all_has_no_loss(orc):
    d = 32
    p = orc.params(d, 1, 4, 1, 1, d, 0.2)
    K = np.random.default_rng(6).standard_normal((10, d))
    cidx, g = orc.channel(p, K, np.ones(d))
    assert np.all(g == 0.0) and np.array_equal(cidx, np.tile(np.arange(d), (10, 1)))


# --------------------------------------------- step 5: top-r and errors


def test_topr_against_full_sort(orc):
    S, r = 64, 8
    p = orc.params(8, 1, S, 1, r, 1, 0.2)
    rng = np.random.default_rng(7)
    for trial in range(50):
        s = rng.integers(0, 6, S).astype(np.float64) if trial % 2 else rng.random(S)
        got = orc.topr(p, s)
        order = np.lexsort((np.arange(S), -s))
        assert np.array_equal(got, np.sort(order[:r]))


def test_segment_errors_hand_values(orc):
    # S=4, r=2: s = (1/2, 1/4, 1/8, 1/8), g = (1/2, 0, 1, 1/4); R = {0, 1}.
    p = orc.params(8, 1, 4, 1, 2, 1, 0.2)
    s = np.array([0.5, 0.25, 0.125, 0.125])
    g = np.array([0.5, 0.0, 1.0, 0.25])
    tidx = orc.topr(p, s)
    assert list(tidx) == [0, 1]
    E = orc.segment_errors(p, s, g, tidx)
    assert list(E) == [0.0, 0.25, 0.25 + 0.125 + 0.03125, 0.25 + 0.25]


# ---------------------------------------------- steps 7-8: hull, budget


def _brute(p, orc, E_all, cap):
    nseg = E_all.shape[0]
    b = [orc.segment_bytes(p, k) for k in range(4)]
    best = None
    for combo in itertools.product(range(4), repeat=nseg):
        by = sum(b[k] for k in combo)
        if by > cap:
            continue
        e = sum(E_all[j, k] for j, k in enumerate(combo))
        if best is None or e < best:
            best = e
    return best


@pytest.mark.parametrize("seed", range(12))
def test_budget_is_optimal_for_its_bytes(orc, seed):
    """Greedy over hull steps stopping at the first misfit is a Lagrangian
    minimiser: no assignment using at most the same bytes has less error."""
    rng = np.random.default_rng(100 + seed)
    S, d = 64, 128
    beta = [0.1, 0.15, 0.2, 0.3, 0.5, 0.9][seed % 6]
    p = orc.params(d, 4, S, 8, 8, 32, beta)
    nseg = 3 + seed % 4
    E_all = np.zeros((nseg, 4))
    for j in range(nseg):
        e_both = rng.random() * 10
        E_all[j] = [0.0, e_both * rng.random(), e_both * rng.random() * 0.8, e_both]
        E_all[j, BOTH] = max(E_all[j, BOTH], E_all[j, TOK], E_all[j, CH])
    st, strat, used = orc.budget(p, E_all)
    Bu = orc.budget_bytes(p, nseg)
    b = [orc.segment_bytes(p, k) for k in range(4)]
    if nseg * min(b) > Bu:
        assert st == 2
        return
    assert st == 0
    assert used == sum(b[k] for k in strat) and used <= Bu
    greedy_e = sum(E_all[j, k] for j, k in enumerate(strat))
    best = _brute(p, orc, E_all, used)
    assert abs(greedy_e - best) <= 1e-12 * max(1.0, abs(best))


def test_budget_each_strategy_wins(orc):
    """Four hand-built segments; under this budget each strategy is the
    optimum of one of them (checked against brute force)."""
    p = orc.params(128, 4, 64, 8, 8, 32, 0.5)
    E_all = np.array([
        [0.0, 5.00, 4.90, 5.10],    # every compression loses a lot -> FULL
        [0.0, 0.001, 3.0, 3.001],   # few heavy tokens -> TOK
        [0.0, 6.00, 0.002, 6.002],  # mass everywhere, channel-sparse -> CH
        [0.0, 0.001, 0.5, 0.0011],  # cheap to drop both ways -> BOTH
    ])
    st, strat, used = orc.budget(p, E_all)
    assert st == 0
    assert list(strat) == [FULL, TOK, CH, BOTH]
    assert abs(sum(E_all[j, k] for j, k in enumerate(strat)) - _brute(p, orc, E_all, used)) < 1e-15


def test_budget_bytes_closed_form(orc):
    """floor(beta * nseg * FULL bytes): 0.3 * 32768 = 9830.4 -> 9830 and
    0.15 * 3 * 32768 = 14745.6 -> 14745 (one rounding, then the floor)."""
    assert orc.budget_bytes(orc.params(128, 4, 64, 8, 8, 32, 0.3), 1) == 9830
    assert orc.budget_bytes(orc.params(128, 4, 64, 8, 8, 32, 0.15), 3) == 14745


def test_budget_equal_efficiency_goes_to_the_lower_segment(orc):
    """Two segments with the same errors have the same hull steps; a budget
    that pays for one upgrade past the cheapest points gives it to segment 0
    (ties in efficiency by the lower segment)."""
    p = orc.params(128, 4, 64, 8, 8, 32, 0.6)
    b = [orc.segment_bytes(p, k) for k in range(4)]       # FULL, TOK, CH, BOTH
    E_all = np.array([[0.0, 0.2, 3.0, 1.0]] * 2)           # hull BOTH -> TOK -> FULL
    verts, _, _ = orc.hull(p, E_all[0])
    assert list(verts) == [BOTH, TOK, FULL]
    nseg = 2
    Bu = orc.budget_bytes(p, nseg)                         # 39321
    assert 2 * b[TOK] + (b[FULL] - b[TOK]) <= Bu < 2 * b[FULL]
    st, strat, used = orc.budget(p, E_all)
    assert st == 0
    # both BOTH -> TOK steps fit; then only one TOK -> FULL step: segment 0's
    assert list(strat) == [FULL, TOK]


def test_budget_beta_one_is_all_full(orc):
    p = orc.params(128, 4, 64, 8, 8, 32, 1.0)
    E_all = np.random.default_rng(9).random((5, 4))
    E_all[:, 0] = 0
    # a segment whose channel-sparse form loses nothing: still FULL at
    # beta = 1 (every segment is kept whole, whatever the errors)
    E_all[2, CH] = 0.0
    st, strat, used = orc.budget(p, E_all)
    assert st == 0 and list(strat) == [FULL] * 5 and used == 5 * 32768


def test_budget_infeasible(orc):
    p = orc.params(128, 4, 64, 8, 8, 32, 0.08)   # 8% < BOTH's 8.64%
    E_all = np.random.default_rng(10).random((4, 4))
    st, _, _ = orc.budget(p, E_all)
    assert st == 2


def test_hull_steps(orc):
    p = orc.params(128, 4, 64, 8, 8, 32, 0.2)
    # CH not better than TOK -> dominated; TOK above the BOTH->FULL chord? no
    verts, eff, db = orc.hull(p, np.array([0.0, 1.0, 2.0, 1.5]))
    assert list(verts) == [BOTH, TOK, FULL]
    assert list(db) == [4112 - 2832, 32768 - 4112]
    assert eff[0] == 0.5 / 1280 and eff[1] == 1.0 / (32768 - 4112)
    # TOK lies above the chord BOTH -> CH -> popped
    verts, _, _ = orc.hull(p, np.array([0.0, 1.999, 0.2, 2.0]))
    assert list(verts) == [BOTH, CH, FULL]
    # an option with the same error as the last hull point and more bytes
    # is no better: TOK (= BOTH) and FULL (= CH) stay off the hull
    verts, _, _ = orc.hull(p, np.array([0.0, 0.5, 0.0, 0.5]))
    assert list(verts) == [BOTH, CH]
    # collinear middle point is popped (the <= in the pop rule)
    b = [32768, 4112, 22528, 2832]
    e_tok = 2.0 - 2.0 * (b[1] - b[3]) / (b[0] - b[3])
    verts, _, _ = orc.hull(p, np.array([0.0, e_tok, 5.0, 2.0]))
    assert list(verts) == [BOTH, FULL]


# --------------------------------------------------------- step 9: pack


def _parse(p, orc, strategy, buf):
    """Independent reader of the packed layout (not the oracle's)."""
    S, d, r, c = p.S, p.d, p.r, p.c
    up = lambda x: -(-x // 16) * 16  # noqa: E731
    o = 0
    tidx = None
    if strategy in (TOK, BOTH):
        tidx = buf[o:o + r].copy()
        o += up(r)
    n = r if strategy in (TOK, BOTH) else S
    if strategy in (FULL, TOK):
        K = buf[o:o + n * d * 2].view(np.uint16).reshape(n, d)
        o += n * d * 2
        cidx = kval = None
    else:
        cidx = buf[o:o + n * c].reshape(n, c)
        o += up(n * c)
        kval = buf[o:o + n * c * 2].view(np.uint16).reshape(n, c)
        o += up(n * c * 2)
        K = None
    V = buf[o:o + n * d * 2].view(np.uint16).reshape(n, d)
    o += n * d * 2
    assert o == len(buf)
    return tidx, K, cidx, kval, V


def test_pack_roundtrip(orc):
    S, d, r, c = 16, 32, 3, 5
    p = orc.params(d, 1, S, 1, r, c, 0.2)
    rng = np.random.default_rng(11)
    K16 = f16(rng.standard_normal((S, d)))
    V16 = f16(rng.standard_normal((S, d)))
    tidx = np.array([2, 7, 11], np.uint8)
    cidx_all = np.array([np.sort(rng.choice(d, c, replace=False)) for _ in range(S)], np.uint8)
    for st in range(4):
        buf = orc.pack_segment(p, st, K16, V16, tidx, cidx_all)
        assert buf.size == orc.segment_bytes(p, st)
        t_, K_, ci_, kv_, V_ = _parse(p, orc, st, buf)
        rows = tidx if st in (TOK, BOTH) else np.arange(S)
        if st in (TOK, BOTH):
            assert np.array_equal(t_, tidx)
        assert np.array_equal(V_, V16.view(np.uint16)[rows])
        if st in (FULL, TOK):
            assert np.array_equal(K_, K16.view(np.uint16)[rows])
        else:
            assert np.array_equal(ci_, cidx_all[rows])
            want = np.take_along_axis(K16.view(np.uint16)[rows], cidx_all[rows].astype(np.int64), 1)
            assert np.array_equal(kv_, want)
        # padding bytes are zero: re-pack into a larger zeroed buffer
        nb = 0
        up = lambda x: -(-x // 16) * 16  # noqa: E731
        if st in (TOK, BOTH):
            assert not buf[r:up(r)].any()
            nb = up(r)
        if st in (CH, BOTH):
            n = r if st == BOTH else S
            assert not buf[nb + n * c: nb + up(n * c)].any()


# ------------------------------------------------------- step 10: decode


def _textbook(q, K, V, scale):
    """fp64 softmax attention through torch's SDPA (library routine)."""
    qt = torch.from_numpy(q)[None, :, None, :]            # [1][G][1][d]
    Kt = torch.from_numpy(K)[None, None].expand(1, q.shape[0], -1, -1)
    Vt = torch.from_numpy(V)[None, None].expand(1, q.shape[0], -1, -1)
    o = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, scale=scale)
    return o[0, :, 0, :].numpy()


def _unit(rng, S, d, G, T, W):
    K16 = f16(rng.standard_normal((T, d)))
    V16 = f16(rng.standard_normal((T, d)))
    qw16 = f16(rng.standard_normal((G * W, d)) + rng.standard_normal(d))
    q16 = f16(rng.standard_normal((G, d)))
    return K16, V16, qw16, q16


def test_decode_full_budget_is_dense_attention(orc):
    S, d, G, W, T = 16, 32, 4, 8, 16 * 7 + 5
    p = orc.params(d, G, S, W, 2, 8, 1.0)
    rng = np.random.default_rng(12)
    K16, V16, qw16, q16 = _unit(rng, S, d, G, T, W)
    res = orc.compress_unit(p, T, 0, K16, V16, qw16)
    assert res["status"] == 0 and np.all(res["strat"] == FULL)
    nc = res["nseg"] * S
    out = orc.decode_unit(p, res["arena"], res["offs"], res["strat"], K16[nc:], V16[nc:], q16)
    ref = _textbook(q16.astype(np.float64), K16.astype(np.float64), V16.astype(np.float64),
                    p.scale)
    assert np.max(np.abs(out - ref)) < 1e-12


def test_decode_keep_everything_strategies_are_dense(orc):
    """TOK with r=S and CH/BOTH with c=d keep every token and channel, so each
    reduces to dense attention."""
    S, d, G = 8, 16, 2
    p = orc.params(d, G, S, 1, S, d, 0.5)
    rng = np.random.default_rng(13)
    nseg = 4
    K16 = f16(rng.standard_normal((nseg * S, d)))
    V16 = f16(rng.standard_normal((nseg * S, d)))
    q16 = f16(rng.standard_normal((G, d)))
    cidx_all = np.tile(np.arange(d, dtype=np.uint8), (S, 1))
    strat = np.array([FULL, TOK, CH, BOTH], np.int32)
    arena, offs = [], []
    o = 0
    for j in range(nseg):
        buf = orc.pack_segment(p, strat[j], K16[j * S:(j + 1) * S], V16[j * S:(j + 1) * S],
                               np.arange(S, dtype=np.uint8), cidx_all)
        offs.append(o)
        arena.append(buf)
        o += buf.size
    out = orc.decode_unit(p, np.concatenate(arena), np.array(offs), strat,
                          K16[:0], V16[:0], q16)
    ref = _textbook(q16.astype(np.float64), K16.astype(np.float64), V16.astype(np.float64),
                    p.scale)
    assert np.max(np.abs(out - ref)) < 1e-12


def test_decode_matches_independent_masked_dense(orc):
    """Second decode path: parse the packed bytes with the test's own reader,
    build the kept keys (dropped channels zeroed) and evaluate softmax
    attention through the library routine."""
    S, d, G, W = 16, 32, 4, 8
    T = S * 9 + 3
    p = orc.params(d, G, S, W, 3, 7, 0.3)
    rng = np.random.default_rng(14)
    K16, V16, qw16, q16 = _unit(rng, S, d, G, T, W)
    res = orc.compress_unit(p, T, 0, K16, V16, qw16)
    assert res["status"] == 0
    assert len(set(res["strat"].tolist())) >= 2
    nc = res["nseg"] * S
    Ks, Vs = [], []
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
        Ks.append(Kd)
        Vs.append(V_.view(np.float16).astype(np.float64))
    Ks.append(K16[nc:].astype(np.float64))
    Vs.append(V16[nc:].astype(np.float64))
    ref = _textbook(q16.astype(np.float64), np.concatenate(Ks), np.concatenate(Vs), p.scale)
    out = orc.decode_unit(p, res["arena"], res["offs"], res["strat"], K16[nc:], V16[nc:], q16)
    assert np.max(np.abs(out - ref)) < 1e-12


def test_decode_over_every_layout_with_sparse_channels(orc):
    """Segments packed as FULL, CH, TOK, BOTH, CH, BOTH with random kept
    tokens and random channel sets (the oracle's own packer, its selection
    steps not involved), plus a dense tail: the decode equals softmax
    attention over the keys the test's parser rebuilds (dropped channels
    zero, each kept value at its own channel)."""
    S, d, G, r, c = 8, 32, 4, 3, 5
    p = orc.params(d, G, S, 8, r, c, 0.3)
    rng = np.random.default_rng(58)
    strat = np.array([FULL, CH, TOK, BOTH, CH, BOTH], np.int32)
    nseg, tail = len(strat), 3
    K16 = f16(rng.standard_normal((nseg * S + tail, d)))
    V16 = f16(rng.standard_normal((nseg * S + tail, d)))
    q16 = f16(rng.standard_normal((G, d)))
    arena, offs, o = [], [], 0
    for j in range(nseg):
        tidx = np.sort(rng.choice(S, r, replace=False)).astype(np.uint8)
        cidx_all = np.stack([np.sort(rng.choice(d, c, replace=False)) for _ in range(S)]).astype(np.uint8)
        buf = orc.pack_segment(p, strat[j], K16[j * S:(j + 1) * S], V16[j * S:(j + 1) * S], tidx, cidx_all)
        offs.append(o)
        arena.append(buf)
        o += buf.size
    arena = np.concatenate(arena)
    Ks, Vs = [], []
    for j in range(nseg):
        end = offs[j + 1] if j + 1 < nseg else o
        t_, K_, ci_, kv_, V_ = _parse(p, orc, int(strat[j]), arena[offs[j]:end])
        n = V_.shape[0]
        if K_ is not None:
            Kd = K_.view(np.float16).astype(np.float64)
        else:
            Kd = np.zeros((n, d))
            for t in range(n):
                Kd[t, ci_[t].astype(np.int64)] = kv_[t].view(np.float16).astype(np.float64)
        Ks.append(Kd)
        Vs.append(V_.view(np.float16).astype(np.float64))
    nc = nseg * S
    Ks.append(K16[nc:].astype(np.float64))
    Vs.append(V16[nc:].astype(np.float64))
    ref = _textbook(q16.astype(np.float64), np.concatenate(Ks), np.concatenate(Vs), p.scale)
    out = orc.decode_unit(p, arena, np.array(offs), strat, K16[nc:], V16[nc:], q16)
    assert np.max(np.abs(out - ref)) < 1e-12


def test_decode_weights_sum_to_one(orc):
    S, d, G, W, T = 16, 32, 2, 4, 16 * 5 + 7
    p = orc.params(d, G, S, W, 2, 4, 0.25)
    rng = np.random.default_rng(15)
    K16, _, qw16, q16 = _unit(rng, S, d, G, T, W)
    V16 = f16(np.ones((T, d)))
    res = orc.compress_unit(p, T, 0, K16, V16, qw16)
    nc = res["nseg"] * S
    out = orc.decode_unit(p, res["arena"], res["offs"], res["strat"], K16[nc:], V16[nc:], q16)
    assert np.max(np.abs(out - 1.0)) < 1e-12


# ----------------------------------------------------- whole compression


def test_keep_all_channels_reduces_to_token_only(orc):
    """c = d: g_t = 0, so CH ties FULL with more bytes and BOTH ties TOK with
    more bytes; the choice must equal the best {FULL, TOK} assignment."""
    S, d, G, W = 16, 16, 2, 4
    T = S * 6
    p = orc.params(d, G, S, W, 4, d, 0.4)
    rng = np.random.default_rng(16)
    K16, V16, qw16, _ = _unit(rng, S, d, G, T, W)
    res = orc.compress_unit(p, T, 0, K16, V16, qw16)
    assert res["status"] == 0
    assert set(res["strat"].tolist()) <= {FULL, TOK}
    assert np.all(res["g"] == 0)
    b = [orc.segment_bytes(p, k) for k in range(4)]
    Bu = orc.budget_bytes(p, res["nseg"])
    best = None
    for combo in itertools.product((FULL, TOK), repeat=res["nseg"]):
        if sum(b[k] for k in combo) > Bu:
            continue
        e = sum(res["E"][j, k] for j, k in enumerate(combo))
        best = e if best is None or e < best else best
    got = sum(res["E"][j, k] for j, k in enumerate(res["strat"]))
    # the greedy may stop short of the budget, but never below the optimum
    # for the bytes it used (checked exactly in the budget tests); here it
    # must also reach the {FULL, TOK} optimum on this instance
    assert got >= best - 1e-12
    best_used = _brute(p, orc, res["E"], res["used"])
    assert abs(got - best_used) < 1e-12


def test_fed_mode_uses_given_scores(orc):
    S, d, G, W, T = 16, 32, 2, 4, 16 * 4
    p = orc.params(d, G, S, W, 3, 8, 0.3)
    rng = np.random.default_rng(17)
    K16, V16, qw16, _ = _unit(rng, S, d, G, T, W)
    a = np.float32(rng.random(d) + 0.5).astype(np.float64)
    s = rng.random(T).astype(np.float32).astype(np.float64)
    res = orc.compress_unit(p, T, 0, K16, V16, qw16, a_in=a, s_in=s)
    assert np.array_equal(res["a"], a) and np.array_equal(res["s"], s)
    for j in range(res["nseg"]):
        assert np.array_equal(res["tidx"][j], orc.topr(p, s[j * S:(j + 1) * S]))


def test_region_offset_matches_shifted_call(orc):
    """Compressing [r0, T) equals compressing a sequence that starts at r0."""
    S, d, G, W = 16, 32, 2, 4
    r0, T = 48, 48 + 16 * 5 + 3
    p = orc.params(d, G, S, W, 3, 8, 0.3)
    rng = np.random.default_rng(18)
    K16, V16, qw16, _ = _unit(rng, S, d, G, T, W)
    a1 = orc.compress_unit(p, T, r0, K16[r0:], V16[r0:], qw16)
    a2 = orc.compress_unit(p, T - r0, 0, K16[r0:], V16[r0:], qw16)
    assert np.array_equal(a1["strat"], a2["strat"])
    assert np.array_equal(a1["arena"], a2["arena"])
    assert np.max(np.abs(a1["s"] - a2["s"])) < 1e-12
