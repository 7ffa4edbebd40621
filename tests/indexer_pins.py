"""Pins of the lightning-indexer oracle (oracle/indexer.py) to facts that do not come from
the oracle itself.

Each pin takes the oracle module ``I`` and raises when it disagrees with what the page
("Ch 04 · CSA", §4 Lightning Indexer) or the mathematics fixes:
* closed forms: one-hot keys make every head's dot product a single query component;
  keys in the negative cone of every head's query score exactly 0 (ReLU);
* identities: the score is linear in the head weights; I(K) - I(-K) equals the
  head-weighted plain dot products, since relu(x) - relu(-x) = x;
* brute force on tiny inputs with exactly rounded sums (math.fsum);
* top-k against its definition checked exhaustively (every selected score is at least
  every unselected one, equal scores go to the smaller index, descending order), and
  the padding when a query has fewer than k candidates.
They run against the real oracle (tests/test_indexer_pins.py) and against broken copies
of it (tests/test_indexer_mutants.py), each of which some pin must reject.
"""

from __future__ import annotations

import math

import numpy as np


def _rand(rng, T, H, D, rows):
    return (rng.standard_normal((T, H, D)), rng.standard_normal((T, H)),
            rng.standard_normal((rows, D)))


def pin_one_hot_keys(I):
    """K_s = e_s: head h's dot product is q[h, s]; the score is sum_h w_h max(0, q[h, s])."""
    rng = np.random.default_rng(1)
    H, D = 5, 9
    q, w = rng.standard_normal((H, D)), rng.standard_normal(H)
    got = I.indexer_scores_row(q, w, np.eye(D))
    for s in range(D):
        want = math.fsum(w[h] * max(0.0, q[h, s]) for h in range(H))
        assert abs(got[s] - want) <= 1e-14 * (1 + abs(want)), (s, got[s], want)


def pin_negative_cone_scores_zero(I):
    """Keys with a negative dot product against every head's query score exactly 0,
    whatever the head weights (ReLU before the weighted sum)."""
    rng = np.random.default_rng(2)
    H, D = 4, 6
    q = np.abs(rng.standard_normal((H, D))) + 0.1      # every query component positive
    K = -np.abs(rng.standard_normal((7, D))) - 0.1     # every key component negative
    w = rng.standard_normal(H) * 10
    got = I.indexer_scores_row(q, w, K)
    assert np.all(got == 0.0), got
    # and keys in the positive cone give the plain weighted sum of dot products
    Kp = -K
    got = I.indexer_scores_row(q, w, Kp)
    for s in range(len(Kp)):
        want = math.fsum(w[h] * math.fsum(q[h, d] * Kp[s, d] for d in range(D)) for h in range(H))
        assert abs(got[s] - want) <= 1e-12 * (1 + abs(want))


def pin_brute_force(I):
    """Every score of a tiny problem against an explicit double loop with fsum."""
    rng = np.random.default_rng(3)
    T, H, D, rows = 3, 3, 5, 11
    q, w, K = _rand(rng, T, H, D, rows)
    key_start = np.array([0, 4, 2])
    n_vis = np.array([11, 7, 0])
    got = I.indexer_scores(q, w, K, key_start, n_vis)
    for t in range(T):
        assert len(got[t]) == n_vis[t]
        for s in range(n_vis[t]):
            key = K[key_start[t] + s]
            want = math.fsum(w[t, h] * max(0.0, math.fsum(q[t, h, d] * key[d] for d in range(D)))
                             for h in range(H))
            assert abs(got[t][s] - want) <= 1e-12 * (1 + abs(want)), (t, s)


def pin_linear_in_head_weights(I):
    rng = np.random.default_rng(4)
    H, D = 6, 8
    q = rng.standard_normal((H, D))
    K = rng.standard_normal((20, D))
    w1, w2 = rng.standard_normal(H), rng.standard_normal(H)
    a = I.indexer_scores_row(q, w1, K)
    b = I.indexer_scores_row(q, w2, K)
    ab = I.indexer_scores_row(q, w1 + w2, K)
    assert np.allclose(ab, a + b, rtol=1e-12, atol=1e-12)
    assert np.allclose(I.indexer_scores_row(q, 3.0 * w1, K), 3.0 * a, rtol=1e-12, atol=1e-12)


def pin_relu_difference_identity(I):
    """relu(x) - relu(-x) = x, so I(K) - I(-K) = sum_h w_h q_h . K."""
    rng = np.random.default_rng(5)
    H, D = 7, 16
    q, w = rng.standard_normal((H, D)), rng.standard_normal(H)
    K = rng.standard_normal((30, D))
    diff = I.indexer_scores_row(q, w, K) - I.indexer_scores_row(q, w, -K)
    want = np.array([math.fsum(w[h] * math.fsum(q[h, d] * K[s, d] for d in range(D))
                               for h in range(H)) for s in range(len(K))])
    assert np.allclose(diff, want, rtol=1e-12, atol=1e-12)


def pin_candidates_are_own_rows(I):
    """Query t scores exactly rows key_start[t] .. key_start[t] + n_visible[t] - 1; rows
    outside the keys are refused."""
    rng = np.random.default_rng(6)
    T, H, D, rows = 4, 2, 3, 40
    q, w, K = _rand(rng, T, H, D, rows)
    ks = np.array([0, 10, 25, 39])
    nv = np.array([10, 15, 15, 1])
    got = I.indexer_scores(q, w, K, ks, nv)
    for t in range(T):
        rows_t = [ks[t] + s for s in range(nv[t])]
        want = [math.fsum(w[t, h] * max(0.0, float(q[t, h] @ K[r])) for h in range(H)) for r in rows_t]
        assert np.allclose(got[t], want, rtol=1e-12, atol=1e-12)
    for bad in ((np.array([35]), np.array([6])), (np.array([-1]), np.array([2]))):
        try:
            I.indexer_scores(q[:1], w[:1], K, *bad)
        except ValueError:
            continue
        raise AssertionError("candidates outside the keys were accepted")


def _check_topk(scores, k, idx, val):
    """The definition, checked exhaustively."""
    S = len(scores)
    n = min(k, S)
    assert len(idx) == k and len(val) == k
    sel = [int(i) for i in idx[:n]]
    assert all(i == -1 for i in idx[n:]) and all(v == -np.inf for v in val[n:])
    assert len(set(sel)) == n and all(0 <= i < S for i in sel)
    chosen = set(sel)
    for i in chosen:
        for j in range(S):
            if j in chosen:
                continue
            assert scores[i] >= scores[j], "a larger score was left out"
            if scores[i] == scores[j]:
                assert i < j, "ties must go to the smaller index"
    for a, b in zip(sel, sel[1:]):
        assert (scores[a] > scores[b]) or (scores[a] == scores[b] and a < b), "order"
    assert all(val[j] == scores[sel[j]] for j in range(n))


def pin_topk_definition(I):
    rng = np.random.default_rng(7)
    for S, k in ((1, 1), (10, 3), (50, 50), (64, 17), (33, 40), (0, 4), (20, 0)):
        # integer scores in a small range: many exact ties, as ReLU zeros make
        scores = rng.integers(-3, 4, size=S).astype(np.float64)
        scores[rng.random(S) < 0.3] = 0.0
        idx, val = I.topk_row(scores, k)
        _check_topk(scores, k, idx, val)
    # continuous scores too
    scores = rng.standard_normal(200)
    _check_topk(scores, 64, *I.topk_row(scores, 64))


def pin_topk_rows(I):
    rows = [np.array([3.0, 1.0, 3.0, 2.0]), np.array([]), np.array([-1.0, 5.0])]
    idx, val = I.indexer_topk(rows, 3)
    assert idx.tolist() == [[0, 2, 3], [-1, -1, -1], [1, 0, -1]]
    assert val[0].tolist() == [3.0, 3.0, 2.0] and val[2][:2].tolist() == [5.0, -1.0]


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
