"""Pins of the oracle's near-tie flags.

The routing is compared with the oracle bit for bit except in rows whose class
boundary is a near tie: the k-th and (k+1)-th pooled probabilities within 1e-5
relative (the tolerance the statement of the method gives for routing). The tie
flags therefore decide which rows leave the exact check, and a flag that were
always set, or compared the wrong positions, would hide routing mismatches.

These tests build layers whose pooled probabilities are chosen by
construction: query block i pools to a unit vector e_h and key block j to
(log w_j, log u_j, 0, 0), so with scale 1 the pooled scores of head h are the
logarithms of chosen weights and their softmax is the weights normalised. Near
ties, clear gaps and ties away from the class boundaries are planted and the
flags are checked against the expected answer of the construction, and, on
random rows, against an all-pairs statement of the same rule.
"""
import math

import numpy as np
import pytest

from oracle import sla_oracle as so

REL = 1e-5  # the routing tie tolerance of the method's statement


class Cfg:
    def __init__(self, **kw):
        base = dict(B=1, H=1, H_kv=1, N=16, N_valid=16, d=4, block=2, mode=0, k_h=2, k_l=2,
                    top_n=0, window=0, causal=0, has_proj=0, proj_per_head=0, has_gate=0,
                    smooth_k=0, linear_all=0, cos_filter=0, scale=1.0, cos_theta=0.0)
        base.update(kw)
        self.__dict__.update(base)


def planted_layer(c, key_logits, query_dirs):
    """Inputs whose pooled key block j is key_logits[j] (a d-vector) and whose pooled
    query block i of head h is query_dirs[h][i] (a d-vector or None = zeros). Each
    block holds two tokens, mean +- a fixed offset, so pooling recovers the vector."""
    nb = c.N // c.block
    assert c.block == 2 and len(key_logits) == nb
    off = np.array([1.0, -1.0, 0.5, -0.5])[:c.d]
    k = np.zeros((1, c.H_kv, c.N, c.d))
    for j, kb in enumerate(key_logits):
        k[0, :, 2 * j] = kb + off
        k[0, :, 2 * j + 1] = kb - off
    q = np.zeros((1, c.H, c.N, c.d))
    for h in range(c.H):
        for i, qb in enumerate(query_dirs[h]):
            if qb is not None:
                q[0, h, 2 * i] = qb + off
                q[0, h, 2 * i + 1] = qb - off
    v = np.zeros((1, c.H_kv, c.N, c.d))
    return so.Layer(c, q, k, v)


def threeway_row(weights, perm, k_h, k_l):
    """Tie flag of query block 0 whose probabilities over the key blocks are
    weights (normalised), placed on the blocks in the order perm."""
    nb = len(weights)
    c = Cfg(N=2 * nb, N_valid=2 * nb, k_h=k_h, k_l=k_l)
    w = np.empty(nb)
    w[np.asarray(perm)] = weights
    keys = [np.array([math.log(x), 0.0, 0.0, 0.0]) for x in w]
    L = planted_layer(c, keys, [[np.array([1.0, 0.0, 0.0, 0.0])] + [None] * (nb - 1)])
    p = so.softmax(L.scores(0, 0)[0])
    np.testing.assert_allclose(p, w / w.sum(), rtol=1e-12)  # the construction holds
    return bool(L.tie_rows(0, 0)[0]), L.classes(0, 0)[0]


PERM8 = [5, 2, 7, 0, 3, 6, 1, 4]  # sorted position -> block index


@pytest.mark.parametrize("weights, expect", [
    ([10, 8, 7, 6, 5, 4, 3, 2], False),                        # clear gaps everywhere
    ([10, 8, 8 * (1 - 5e-6), 6, 5, 4, 3, 2], True),            # k_h boundary (positions 1 | 2)
    ([10, 8, 8 * (1 - 0.9e-5), 6, 5, 4, 3, 2], True),          # just inside the tolerance
    ([10, 8, 8 * (1 - 2e-5), 6, 5, 4, 3, 2], False),           # just outside it
    ([10, 8, 7, 6, 5, 4, 4 * (1 - 5e-6), 2], True),            # k_l boundary (positions 5 | 6)
    ([10, 8, 7, 6, 5, 4, 4 * (1 - 2e-5), 2], False),
    ([10, 8, 7, 6, 6 * (1 - 5e-6), 4, 3, 2], False),           # tie between two marginal blocks
    ([10, 10 * (1 - 5e-6), 7, 6, 5, 4, 3, 2], False),          # tie between two critical blocks
    ([10, 8, 7, 6, 5, 4, 3, 3 * (1 - 5e-6)], False),           # tie between two negligible blocks
])
def test_threeway_tie_flag_planted(weights, expect):
    tie, cls = threeway_row(np.array(weights, float), PERM8, k_h=2, k_l=2)
    assert tie == expect
    # the classes follow the sorted positions regardless of the flag
    crit = sorted(PERM8[:2]); neg = sorted(PERM8[-2:])
    assert sorted(np.nonzero(cls == so.CRITICAL)[0].tolist()) == crit
    assert sorted(np.nonzero(cls == so.NEGLIGIBLE)[0].tolist()) == neg


def test_threeway_tie_flag_without_negligible_blocks_ignores_the_last_position():
    # k_l = 0: only the k_h boundary exists; a near tie at the bottom is not a boundary
    w = np.array([10, 8, 7, 6, 5, 4, 3, 3 * (1 - 5e-6)], float)
    assert threeway_row(w, PERM8, k_h=2, k_l=0)[0] is False
    w = np.array([10, 8, 8 * (1 - 5e-6), 6, 5, 4, 3, 2], float)
    assert threeway_row(w, PERM8, k_h=2, k_l=0)[0] is True


def test_threeway_tie_flag_all_or_nothing_critical_has_no_boundary():
    w = np.array([10, 10, 10, 10, 10, 10, 10, 10], float)  # every pair is an exact tie
    assert threeway_row(w, PERM8, k_h=8, k_l=0)[0] is False  # no block is left out
    assert threeway_row(w, PERM8, k_h=0, k_l=0)[0] is False
    assert threeway_row(w, PERM8, k_h=0, k_l=8)[0] is False
    assert threeway_row(w, PERM8, k_h=3, k_l=0)[0] is True


def brute_threeway_tie(p, k_h, k_l, rel=REL):
    """All pairs: a row is a near tie when some block inside a class and some block
    outside it, across either class boundary, have probabilities within rel."""
    nb = len(p)
    order = sorted(range(nb), key=lambda j: (-p[j], j))
    tie = False
    for cut in (k_h, nb - k_l):
        if not 0 < cut < nb:
            continue
        inside, outside = order[:cut], order[cut:]
        for a in inside:
            for b in outside:
                if abs(p[a] - p[b]) <= rel * max(p[a], p[b]):
                    tie = True
    return tie


def test_threeway_tie_flags_match_all_pairs_on_random_rows():
    rng = np.random.default_rng(11)
    nb, seen = 12, {True: 0, False: 0}
    for trial in range(60):
        w = rng.uniform(1.0, 2.0, nb)
        k_h, k_l = int(rng.integers(1, 5)), int(rng.integers(0, 5))
        order = np.argsort(-w, kind="stable")
        if trial % 3 == 0:    # a near tie (or just not one) across a class boundary
            cut = k_h if trial % 2 == 0 or k_l == 0 else nb - k_l
            a, b = order[cut - 1], order[cut]
            w[b] = w[a] * (1 - rng.uniform(0, 2e-5))
        elif trial % 3 == 1:  # between two random blocks
            a, b = rng.choice(nb, 2, replace=False)
            w[b] = w[a] * (1 - rng.uniform(0, 2e-5))
        c = Cfg(N=2 * nb, N_valid=2 * nb, k_h=k_h, k_l=k_l)
        keys = [np.array([math.log(x), 0.0, 0.0, 0.0]) for x in w]
        L = planted_layer(c, keys, [[np.array([1.0, 0.0, 0.0, 0.0])] + [None] * (nb - 1)])
        p = so.softmax(L.scores(0, 0)[0])
        got = bool(L.tie_rows(0, 0)[0])
        assert got == brute_threeway_tie(p, k_h, k_l), (trial, w, k_h, k_l)
        seen[got] += 1
    assert seen[True] >= 5 and seen[False] >= 5  # both outcomes are exercised


# ---------------------------------------------------------------------------
# top-n mode: the group's summed probabilities decide the selection and the tie
# ---------------------------------------------------------------------------
P_HEAD0 = np.array([0.30, 0.10, 0.15, 0.25, 0.12, 0.08])
PERM6 = [4, 0, 5, 2, 1, 3]   # value index -> block index (blocks 0..5 are the candidates of block 6)


def topn_row(group_sum, top_n=3, perm=PERM6):
    """Query block 6 of a group of two heads whose per-head probabilities over the
    candidates j < 6 are P_HEAD0 and group_sum - P_HEAD0. Returns (selected, tie)."""
    r = np.asarray(group_sum, float) - P_HEAD0
    assert abs(r.sum() - 1) < 1e-12 and (r > 0).all()
    c = Cfg(H=2, H_kv=1, N=16, N_valid=16, mode=1, k_h=0, k_l=0, top_n=top_n, causal=1)
    nb = 8
    keys = [np.zeros(4) for _ in range(nb)]
    for idx, j in enumerate(perm):
        keys[j] = np.array([math.log(P_HEAD0[idx]), math.log(r[idx]), 0.0, 0.0])
    dirs = [[None] * 6 + [np.array([1.0, 0, 0, 0]), None], [None] * 6 + [np.array([0, 1.0, 0, 0]), None]]
    L = planted_layer(c, keys, dirs)
    sel, tie = L.selection(0, 0)
    return sel[6].tolist(), bool(tie[6])


def sums_with(pos3):
    """Group sums with a chosen value at sorted position 3 (the one just outside a top 3);
    the last entry absorbs the change so the sums stay a valid pair of distributions."""
    s = np.array([0.50, 0.45, 0.40, pos3, 0.15, 0.0])
    s[5] = 2.0 - s[:5].sum()
    return s


def test_topn_tie_flag_uses_the_group_sum_at_the_selection_boundary():
    # each head alone has a clear gap at position 3; only the sum ties there
    s = sums_with(0.40 * (1 - 5e-6))
    r = s - P_HEAD0
    for p in (P_HEAD0, r):
        o = np.sort(p)[::-1]
        assert (o[2] - o[3]) / o[2] > 1e-2
    sel, tie = topn_row(s)
    assert tie is True
    assert sel == sorted(PERM6[:3])


@pytest.mark.parametrize("pos3, expect", [
    (0.40 * (1 - 0.9e-5), True),
    (0.40 * (1 - 2e-5), False),
    (0.30, False),
])
def test_topn_tie_flag_threshold(pos3, expect):
    sel, tie = topn_row(sums_with(pos3))
    assert tie == expect
    assert sel == sorted(PERM6[:3])


def test_topn_tie_away_from_the_boundary_is_not_flagged():
    s = np.array([0.50, 0.50 * (1 - 5e-6), 0.40, 0.30, 0.15, 0.0])  # tie inside the selection
    s[5] = 2.0 - s[:5].sum()
    assert topn_row(s)[1] is False
    x = 0.175 / (1 - 2.5e-6)                                         # tie outside it (positions 4 | 5)
    s = np.array([0.50, 0.45, 0.40, 0.30, x, x * (1 - 5e-6)])
    assert abs(s.sum() - 2.0) < 1e-12 and abs(s[4] - s[5]) <= REL * s[4]
    assert topn_row(s)[1] is False


def test_topn_tie_flag_when_every_candidate_is_selected():
    s = sums_with(0.40 * (1 - 5e-6))
    sel, tie = topn_row(s, top_n=6)  # all six candidates fit: no boundary
    assert tie is False and sel == list(range(6))
    sel, tie = topn_row(s, top_n=4)  # the boundary moves to positions 3 | 4: clear
    assert tie is False and sel == sorted(PERM6[:4])


# ---------------------------------------------------------------------------
# planted mistakes: a tie rule that flags every row, or compares the wrong
# positions, fails the pins above
# ---------------------------------------------------------------------------
def _expect_pin_failure(fn, *args):
    with pytest.raises(AssertionError):
        fn(*args)


def test_planted_always_flagged_threeway_rows_are_caught(monkeypatch):
    monkeypatch.setattr(so, "threeway_tie_rows", lambda s, k_h, k_l, rel=REL: np.ones(s.shape[0], bool))
    _expect_pin_failure(test_threeway_tie_flag_planted, [10, 8, 7, 6, 5, 4, 3, 2], False)


def test_planted_shifted_threeway_boundary_is_caught(monkeypatch):
    def shifted(scores, k_h, k_l, rel=REL):  # compares positions k and k+1 instead of k-1 and k
        p = so.softmax(scores)
        nb = scores.shape[1]
        tie = np.zeros(scores.shape[0], bool)
        for i in range(scores.shape[0]):
            o = so.block_order(scores[i])
            for pos in (k_h, nb - k_l):
                if 0 < pos < nb - 1:
                    a, b = p[i, o[pos]], p[i, o[pos + 1]]
                    tie[i] |= abs(a - b) <= rel * max(a, b)
        return tie
    monkeypatch.setattr(so, "threeway_tie_rows", shifted)
    _expect_pin_failure(test_threeway_tie_flag_planted, [10, 8, 8 * (1 - 5e-6), 6, 5, 4, 3, 2], True)


def test_planted_topn_tie_on_one_head_only_is_caught(monkeypatch):
    real = so.select_topn

    def first_head_only(group_scores, top_n, rel=REL):  # the tie taken from head 0's probabilities
        sel, _ = real(group_scores, top_n, rel)
        _, tie = real(group_scores[:1], top_n, rel)
        return sel, tie
    monkeypatch.setattr(so, "select_topn", first_head_only)
    _expect_pin_failure(test_topn_tie_flag_uses_the_group_sum_at_the_selection_boundary)
