"""Pins of the oracle's Token2Chunk selection (Kara, "What carries the
argument": chunks between high-score tokens under a length cap and a
budget) against facts that do not come from its own arithmetic: the
parameter settings that reduce it to plain top-r, a closed form for
all-equal scores, hand-worked examples, and structural invariants on random
segments."""
import numpy as np
import pytest


def _p(orc, S, r, gamma, alpha):
    return orc.params(128, 4, S, 8, r, 32, 0.3, chunk_len=gamma, chunk_budget=alpha)


def test_no_budget_or_no_room_is_plain_top_r(orc):
    rng = np.random.default_rng(41)
    for _ in range(50):
        S, r = 64, 8
        s = rng.random(S)
        s[rng.choice(S, 5)] = 0.5            # some ties
        plain = orc.topr(orc.params(128, 4, S, 8, r, 32, 0.3), s)
        # alpha = 0: the core is already r tokens
        assert np.array_equal(orc.topr_chunks(_p(orc, S, r, 8, 0), s), plain)
        # gamma = 2: no gap can be filled, the budget goes to the next best
        assert np.array_equal(orc.topr_chunks(_p(orc, S, r, 2, 4), s), plain)


def test_equal_scores_keep_the_first_r(orc):
    # ties go to the lower token: the core is 0..r-alpha-1 (no gaps), the
    # remaining budget takes the next lowest tokens
    s = np.full(32, 0.25)
    assert orc.topr_chunks(_p(orc, 32, 6, 8, 3), s).tolist() == [0, 1, 2, 3, 4, 5]


def test_hand_worked_gap_fill_and_skip(orc):
    # S = 16, r = 6, alpha = 3, gamma = 5.  Core (top 3): tokens 2, 5, 11
    # (scores 9, 8, 7).  Gaps: (2, 5) holds 3, 4 (span 4 <= 5, merit
    # 0.4 + 0.3 = 0.7); (5, 11) spans 7 > 5: not a candidate.  Fill 3, 4
    # (budget 3 -> 1); the last token is the best left: 13 (0.6).
    s = np.zeros(16)
    s[[2, 5, 11]] = [9.0, 8.0, 7.0]
    s[3], s[4] = 0.4, 0.3
    s[13] = 0.6
    s[0] = 0.5
    assert orc.topr_chunks(_p(orc, 16, 6, 5, 3), s).tolist() == [2, 3, 4, 5, 11, 13]


def test_hand_worked_merit_order_and_budget_skip(orc):
    # S = 32, r = 7, alpha = 3, gamma = 6.  Core (top 4): 1, 4, 8, 10.
    # Candidates: (1, 4) gap 2 (tokens 2, 3; merit 0.2), (4, 8) gap 3
    # (5, 6, 7; merit 0.9), (8, 10) gap 1 (token 9; merit 0.25).  By merit:
    # (4, 8) fits (3 <= 3, budget -> 0); the others no longer fit.
    s = np.zeros(32)
    s[[1, 4, 8, 10]] = [5.0, 4.0, 3.0, 2.0]
    s[2], s[3] = 0.1, 0.1
    s[5], s[6], s[7] = 0.3, 0.3, 0.3
    s[9] = 0.25
    s[20] = 1.0                              # the best non-core token, not needed
    assert orc.topr_chunks(_p(orc, 32, 7, 6, 3), s).tolist() == [1, 4, 5, 6, 7, 8, 10]
    # with budget 2 the merit-0.9 gap (3 tokens) is skipped, the 0.25 gap
    # (1 token, start 8) then the 0.2 gap (2 tokens) no longer fits: the
    # last token is the best left (20)
    assert orc.topr_chunks(_p(orc, 32, 6, 6, 2), s).tolist() == [1, 4, 8, 9, 10, 20]


def test_hand_worked_span_cap_is_inclusive(orc):
    # S = 16, r = 6, alpha = 3.  Core (top 3): tokens 2, 6, 12.  The chunk
    # from 2 to 6 holds the gap 3, 4, 5 and spans 6 - 2 + 1 = 5 tokens,
    # endpoints included; (6, 12) spans 7.  With gamma = 5 the first gap is
    # a candidate and fills the whole budget: 2, 3, 4, 5, 6, 12.  With
    # gamma = 4 neither gap is, and the budget goes to the best tokens left:
    # 14, 0, 15.
    s = np.zeros(16)
    s[[2, 6, 12]] = [9.0, 8.0, 7.0]
    s[3], s[4], s[5] = 0.1, 0.1, 0.1
    s[14], s[0], s[15] = 0.9, 0.8, 0.7
    assert orc.topr_chunks(_p(orc, 16, 6, 5, 3), s).tolist() == [2, 3, 4, 5, 6, 12]
    assert orc.topr_chunks(_p(orc, 16, 6, 4, 3), s).tolist() == [0, 2, 6, 12, 14, 15]


def test_hand_worked_equal_merits_go_to_the_lower_gap(orc):
    # S = 16, r = 5, alpha = 1, gamma = 3.  Core (top 4): 1, 3, 9, 11.  Gaps
    # (1, 3) and (9, 11) hold one token each (2 and 10) with the same merit
    # 0.5; the budget of 1 fills the one that starts lower: token 2.
    s = np.zeros(16)
    s[[1, 3, 9, 11]] = [9.0, 8.0, 7.0, 6.0]
    s[2] = s[10] = 0.5
    s[14] = 0.9
    assert orc.topr_chunks(_p(orc, 16, 5, 3, 1), s).tolist() == [1, 2, 3, 9, 11]


@pytest.mark.parametrize("seed", range(6))
def test_structure_on_random_segments(orc, seed):
    rng = np.random.default_rng(100 + seed)
    S, r, alpha, gamma = 64, 8, 4, 8
    s = rng.random(S) ** 3
    s[rng.choice(S, 6)] = s[0]               # ties
    t = orc.topr_chunks(_p(orc, S, r, gamma, alpha), s)
    assert len(t) == r and np.all(np.diff(t.astype(int)) > 0)
    order = np.lexsort((np.arange(S), -s))
    core = set(order[:r - alpha].tolist())
    kept = set(t.tolist())
    assert core <= kept
    extra = sorted(kept - core)
    # the extra tokens are whole gaps between consecutive core tokens of span
    # <= gamma (chunks, at most alpha tokens in all), and the best tokens
    # left after core and chunks
    cs = sorted(core)
    gaps = [(a, b) for a, b in zip(cs, cs[1:]) if b - a - 1 >= 1 and b - a + 1 <= gamma]
    whole = [g for g in gaps if all(x in kept for x in range(g[0] + 1, g[1]))]
    chunk = [x for a, b in whole for x in range(a + 1, b)]
    assert len(chunk) <= alpha
    rest = [x for x in extra if x not in chunk]
    best_left = [x for x in order.tolist() if x not in core and x not in chunk][:len(rest)]
    assert sorted(rest) == sorted(best_left)
