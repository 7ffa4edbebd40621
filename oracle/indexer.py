"""fp64 CPU oracle of the lightning indexer: scores over compressed indexer keys and the
top-k selection that follows them.

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
cpu_baseline / reference legs may import or run this module.  The product package
(``kv_token_compressor_b200``) never imports it and shares no code with it.

What it follows (page "Ch 04 · CSA", §4 "Lightning Indexer", the score equation and the
selected-set equation; §5 for k):

* Score of query t against compressed indexer key s: every indexer head h takes the dot
  product of its query q^I_{t,h} with the key K^{IComp}_s, passes it through ReLU, and the
  heads are summed with the per-query head weights w^I_{t,h}:
      I[t, s] = sum_h w[t, h] * max(0, q[t, h] . K[s]).
  One key per entry is shared by all heads (multi-query).  Sizes on the page: 64 heads,
  key width c^I = 128.
* Selection: the entries whose scores are among the k largest of the query's candidates
  (k = 1024 on the Pro model, 512 on Flash).

Readings where the page is silent:
* Candidates: query t scores the n_visible[t] keys K[key_start[t] : key_start[t] +
  n_visible[t]] of its own sequence (a decode step sees all of its sequence's entries; a
  prefill query only the entries whose blocks are complete -- the caller decides).
* Order and ties: the selection is returned in descending score order, equal scores by
  ascending entry index, so the selected set and its order are unique; when a query has
  fewer than k candidates, all of them are returned and the rest is padded with -1.

All array arguments are widened exactly to float64 (bf16 and fp32 values are exactly
representable in float64); the dot products are float64 sums.
"""

from __future__ import annotations

import numpy as np

__all__ = ["indexer_scores_row", "indexer_scores", "topk_row", "indexer_topk"]


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def indexer_scores_row(q_t, w_t, K_rows):
    """Scores of one query against its candidate keys ("Ch 04 · CSA", §4, score equation).

    q_t: [H, D] queries of the query's heads; w_t: [H] head weights; K_rows: [S, D] the
    candidate keys.  Returns [S] float64: sum_h w_t[h] * max(0, q_t[h] . K_rows[s]).
    """
    q = _f64(q_t)
    w = _f64(w_t)
    K = _f64(K_rows)
    if q.ndim != 2 or K.ndim != 2 or q.shape[1] != K.shape[1] or w.shape != (q.shape[0],):
        raise ValueError("shapes: q [H, D], w [H], K [S, D]")
    dots = K @ q.T                      # [S, H]: head h's inner product with each key
    relu = np.maximum(dots, 0.0)        # negative correlations count as zero
    return relu @ w                     # head-weighted sum


def indexer_scores(q, w, K, key_start, n_visible):
    """Scores of every query over its own candidates.

    q [T, H, D], w [T, H], K [rows, D] (the compressed indexer keys of all sequences,
    packed), key_start / n_visible [T] integers.  Returns a list of T float64 arrays, the
    t-th of length n_visible[t].
    """
    q = _f64(q)
    w = _f64(w)
    out = []
    for t in range(q.shape[0]):
        s0, nv = int(key_start[t]), int(n_visible[t])
        if s0 < 0 or nv < 0 or s0 + nv > len(K):
            raise ValueError(f"query {t}: candidates [{s0}, {s0 + nv}) outside the keys")
        out.append(indexer_scores_row(q[t], w[t], K[s0:s0 + nv]))
    return out


def topk_row(scores, k: int):
    """Indices of the k largest scores ("Ch 04 · CSA", §4, selected-set equation), in
    descending score order with equal scores by ascending index; padded with -1 when
    there are fewer than k candidates.  Returns (indices int64 [k], scores float64 [k],
    padded with -inf)."""
    s = _f64(scores)
    if k < 0:
        raise ValueError("k >= 0")
    order = sorted(range(len(s)), key=lambda i: (-s[i], i))[:k]
    idx = np.full(k, -1, dtype=np.int64)
    val = np.full(k, -np.inf)
    idx[:len(order)] = order
    val[:len(order)] = s[order]
    return idx, val


def indexer_topk(score_rows, k: int):
    """topk_row for every query's score row; returns ([T, k] int64, [T, k] float64)."""
    res = [topk_row(r, k) for r in score_rows]
    if not res:
        return np.zeros((0, k), dtype=np.int64), np.zeros((0, k))
    return np.stack([r[0] for r in res]), np.stack([r[1] for r in res])
