"""Pins of the fp64 oracle to facts that do not come from the oracle itself.

Each pin takes the oracle module ``O`` and raises AssertionError (or any exception)
when the oracle disagrees with what the pages or the mathematics fix.  The pins are
run against the real oracle (tests/test_oracle_pins.py) and against deliberately
broken copies of it (tests/test_oracle_mutants.py), which every pin set must reject.

Sources of truth used here, none of them the oracle's own code:
* the 12-token worked example of "Ch 04 · CSA" §3 (tests/golden/csa_worked_example_m4_n12.json);
* the entry counts of "序列压缩注意力" table attn-seqcomp-csa-hca and "Ch 05 · HCA"
  (tests/golden/entry_counts.json);
* the coverage identity of table attn-seqcomp-overlap and the entry-0 boundary of
  eq. attn-seqcomp-overlap-bound ("序列压缩注意力");
* closed forms: the mean (constant logits), the logistic function (a two-row softmax),
  one-hot limits, convexity, linearity in C, shift invariance of the softmax;
* library routines: scipy.special.softmax, math.fsum dot products.
"""

from __future__ import annotations

import json
import math
import os

import numpy as np

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _rand_csa(rng, batch, n, c, m):
    f = lambda *s: rng.standard_normal(s)
    return dict(Ca=f(batch, n, c), Cb=f(batch, n, c), Za=f(batch, n, c), Zb=f(batch, n, c),
                Ba=0.3 * f(m, c), Bb=0.3 * f(m, c))


def _csa(O, d, m, overlap=True, entries=None):
    return O.csa_compress(d["Ca"], d["Cb"], d["Za"], d["Zb"], d["Ba"], d["Bb"], m, overlap,
                          entries=entries)


def _fsum_pool(L, V):
    """Independent evaluation: scipy's softmax over rows and exactly rounded sums."""
    from scipy.special import softmax

    S = softmax(np.asarray(L, np.float64), axis=0)
    V = np.asarray(V, np.float64)
    return np.array([math.fsum(S[:, ch] * V[:, ch]) for ch in range(V.shape[1])])


# --------------------------------------------------------------------------------------
# Indexing (bit-exact)
# --------------------------------------------------------------------------------------

def pin_entry_counts(O):
    g = _load("entry_counts.json")
    for case in g["exact"]:
        assert O.num_entries(case["n"], case["m"]) == case["entries"], case
    for case in g["approx"]:
        got = O.num_entries(case["n"], case["m"])
        assert abs(got - case["page_value"]) <= case["rel_tol"] * case["page_value"], (case, got)
    # The pages' 1M contexts are binary 2^20 in the workloads: exact quotients.
    assert O.num_entries(1 << 20, 4) == 262144
    assert O.num_entries(1 << 20, 128) == 8192
    # Incomplete trailing block is not an entry.
    for n in range(0, 40):
        for m in (1, 2, 3, 4, 8):
            ne = O.num_entries(n, m)
            assert ne * m <= n < (ne + 1) * m, (n, m, ne)


def pin_coverage_identity(O):
    for m in (1, 2, 4, 8, 128):
        for i in range(0, 50):
            a_i, b_i = O.entry_rows(i, m)
            a_next, b_next = O.entry_rows(i + 1, m)
            assert list(a_i) == list(b_next), (m, i)
            assert len(a_i) == m and len(b_i) == m
            assert a_i.start == m * i
        _, b0 = O.entry_rows(0, m)
        assert list(b0) == list(range(-m, 0))


def pin_worked_example_dependencies(O):
    """Perturb every row of every stream; the entries that change must be exactly those
    the worked example says read that row."""
    g = _load("csa_worked_example_m4_n12.json")
    n, m = g["n"], g["m"]
    rng = np.random.default_rng(11)
    c = 3
    d = _rand_csa(rng, 1, n, c, m)
    base = _csa(O, d, m)
    assert base.shape == (1, g["num_entries"], c)
    reads = {"a": {}, "b": {}}
    for e in g["entries"]:
        for part in ("a", "b"):
            rr = e[part + "_rows"]
            if rr is not None:
                for r in range(rr[0], rr[1] + 1):
                    reads[part].setdefault(r, set()).add(e["i"])
    for stream, part in (("Ca", "a"), ("Za", "a"), ("Cb", "b"), ("Zb", "b")):
        for r in range(n):
            d2 = {k: v.copy() for k, v in d.items()}
            d2[stream][0, r] += rng.standard_normal(c) + 0.5
            out = _csa(O, d2, m)
            changed = {i for i in range(g["num_entries"]) if not np.array_equal(out[0, i], base[0, i])}
            assert changed == reads[part].get(r, set()), (stream, r, changed)
    x4 = g["token_x4"]
    a_in = {e["i"] for e in g["entries"] if e["a_rows"] and e["a_rows"][0] <= 4 <= e["a_rows"][1]}
    b_in = {e["i"] for e in g["entries"] if e["b_rows"] and e["b_rows"][0] <= 4 <= e["b_rows"][1]}
    assert a_in == {x4["enters_by_stream_a"]} and b_in == {x4["enters_by_stream_b"]}


# --------------------------------------------------------------------------------------
# Softmax / pool closed forms
# --------------------------------------------------------------------------------------

def pin_entry0_is_pure_a(O):
    rng = np.random.default_rng(1)
    for m in (1, 4, 8):
        d = _rand_csa(rng, 2, 5 * m, 6, m)
        out = _csa(O, d, m)
        for b in range(2):
            ref = _fsum_pool(d["Za"][b, :m] + d["Ba"], d["Ca"][b, :m])
            assert np.allclose(out[b, 0], ref, rtol=1e-13, atol=1e-13)
        d2 = dict(d)
        d2["Cb"] = rng.standard_normal(d["Cb"].shape) * 100
        d2["Zb"] = rng.standard_normal(d["Zb"].shape) * 100
        d2["Bb"] = rng.standard_normal(d["Bb"].shape) * 100
        out2 = _csa(O, d2, m)
        assert np.array_equal(out2[:, 0], out[:, 0])


def pin_weights_sum_to_one(O):
    rng = np.random.default_rng(2)
    for m in (1, 4):
        d = _rand_csa(rng, 1, 6 * m, 5, m)
        d["Ca"][:] = 1.0
        d["Cb"][:] = 1.0
        assert np.allclose(_csa(O, d, m), 1.0, rtol=0, atol=1e-14)
    C = np.ones((2, 256, 4))
    Z = rng.standard_normal((2, 256, 4)) * 5
    B = rng.standard_normal((128, 4))
    assert np.allclose(O.hca_compress(C, Z, B, 128), 1.0, rtol=0, atol=1e-14)


def pin_mean_pooling(O):
    """Constant logits and zero bias: every weight is 1/rows, the entry is the mean."""
    rng = np.random.default_rng(3)
    m, ne, c = 4, 6, 5
    d = _rand_csa(rng, 1, m * ne, c, m)
    d["Za"][:] = 0.7
    d["Zb"][:] = 0.7
    d["Ba"][:] = 0.0
    d["Bb"][:] = 0.0
    out = _csa(O, d, m)
    for i in range(ne):
        for ch in range(c):
            vals = list(d["Ca"][0, m * i:m * i + m, ch])
            if i > 0:
                vals += list(d["Cb"][0, m * (i - 1):m * i, ch])
            assert abs(out[0, i, ch] - math.fsum(vals) / len(vals)) < 1e-14
    # HCA: the "simple average" of a 128-token segment.
    C = rng.standard_normal((1, 384, c))
    Z = np.full((1, 384, c), -2.5)
    B = np.zeros((128, c))
    out = O.hca_compress(C, Z, B, 128)
    for i in range(3):
        for ch in range(c):
            assert abs(out[0, i, ch] - math.fsum(C[0, 128 * i:128 * i + 128, ch]) / 128) < 1e-14


def pin_shift_invariance(O):
    rng = np.random.default_rng(4)
    m = 4
    d = _rand_csa(rng, 1, 32, 6, m)
    base = _csa(O, d, m)
    s = rng.standard_normal(6) * 3
    d2 = dict(d, Za=d["Za"] + s, Zb=d["Zb"] + s, Ba=d["Ba"] + 1.25, Bb=d["Bb"] + 1.25)
    assert np.allclose(_csa(O, d2, m), base, rtol=1e-12, atol=1e-12)


def pin_one_hot_logit(O):
    """A row whose logit is +60 above the rest takes all the weight: the entry that
    reads it equals that row's vector (brute force over every row of both streams)."""
    rng = np.random.default_rng(5)
    m, ne, c = 4, 4, 3
    n = m * ne
    d = _rand_csa(rng, 1, n, c, m)
    for r in range(n):
        for zs, cs, target in (("Za", "Ca", r // m), ("Zb", "Cb", r // m + 1)):
            if target >= ne:
                continue
            d2 = {k: v.copy() for k, v in d.items()}
            d2[zs][0, r] += 60.0
            out = _csa(O, d2, m, entries=[(0, target)])
            assert np.allclose(out[0], d[cs][0, r], rtol=1e-12, atol=1e-12), (zs, r)


def pin_bias_one_hot(O):
    """B^a[k] (or B^b[k]) far above the rest selects in-block position k of the a-block
    (or of the previous block through stream b) in every entry."""
    rng = np.random.default_rng(6)
    m, ne, c = 4, 5, 3
    d = _rand_csa(rng, 1, m * ne, c, m)
    for k in range(m):
        d2 = {kk: v.copy() for kk, v in d.items()}
        d2["Ba"][k] += 60.0
        out = _csa(O, d2, m)
        for i in range(ne):
            assert np.allclose(out[0, i], d["Ca"][0, m * i + k], rtol=1e-12, atol=1e-12), (k, i)
        d3 = {kk: v.copy() for kk, v in d.items()}
        d3["Bb"][k] += 60.0
        out = _csa(O, d3, m)
        for i in range(1, ne):
            assert np.allclose(out[0, i], d["Cb"][0, m * (i - 1) + k], rtol=1e-12, atol=1e-12), (k, i)
        assert np.allclose(out[0, 0], _fsum_pool(d["Za"][0, :m] + d["Ba"], d["Ca"][0, :m]),
                           rtol=1e-13, atol=1e-13)
    # HCA bias one-hot
    C = rng.standard_normal((1, 256, c))
    Z = rng.standard_normal((1, 256, c))
    for k in (0, 77, 127):
        B = rng.standard_normal((128, c)) * 0.1
        B[k] += 60.0
        out = O.hca_compress(C, Z, B, 128)
        for i in range(2):
            assert np.allclose(out[0, i], C[0, 128 * i + k], rtol=1e-12, atol=1e-12)


def pin_two_row_logistic(O):
    """m = 1 with overlap: a two-row softmax is the logistic function,
    out_i = s ca_i + (1 - s) cb_{i-1}, s = 1 / (1 + exp(-(za_i + ba - zb_{i-1} - bb)))."""
    rng = np.random.default_rng(7)
    n, c = 9, 4
    d = _rand_csa(rng, 1, n, c, 1)
    out = _csa(O, d, 1)
    for i in range(n):
        for ch in range(c):
            if i == 0:
                ref = d["Ca"][0, 0, ch]
            else:
                x = d["Za"][0, i, ch] + d["Ba"][0, ch] - d["Zb"][0, i - 1, ch] - d["Bb"][0, ch]
                s = 1.0 / (1.0 + math.exp(-x))
                ref = s * d["Ca"][0, i, ch] + (1.0 - s) * d["Cb"][0, i - 1, ch]
            assert abs(out[0, i, ch] - ref) < 1e-14, (i, ch)


def pin_library_softmax(O):
    """Every entry against scipy.special.softmax over the rows the pages name, with
    exactly rounded weighted sums (CSA m = 4 overlap and HCA m' = 128)."""
    rng = np.random.default_rng(8)
    m, ne, c = 4, 6, 7
    d = _rand_csa(rng, 1, m * ne + 3, c, m)
    d["Za"] *= 3
    out = _csa(O, d, m)
    assert out.shape == (1, ne, c)
    for i in range(ne):
        La = d["Za"][0, m * i:m * i + m] + d["Ba"]
        Va = d["Ca"][0, m * i:m * i + m]
        if i == 0:
            ref = _fsum_pool(La, Va)
        else:
            Lb = d["Zb"][0, m * (i - 1):m * i] + d["Bb"]
            Vb = d["Cb"][0, m * (i - 1):m * i]
            ref = _fsum_pool(np.vstack([La, Lb]), np.vstack([Va, Vb]))
        assert np.allclose(out[0, i], ref, rtol=1e-13, atol=1e-13), i
    C = rng.standard_normal((2, 300, c))
    Z = rng.standard_normal((2, 300, c)) * 4
    B = rng.standard_normal((128, c))
    out = O.hca_compress(C, Z, B, 128)
    assert out.shape == (2, 2, c)
    for b in range(2):
        for i in range(2):
            ref = _fsum_pool(Z[b, 128 * i:128 * i + 128] + B, C[b, 128 * i:128 * i + 128])
            assert np.allclose(out[b, i], ref, rtol=1e-13, atol=1e-13)


def pin_convexity(O):
    rng = np.random.default_rng(9)
    m, ne, c = 4, 8, 16
    d = _rand_csa(rng, 1, m * ne, c, m)
    d["Za"] *= 6
    d["Zb"] *= 6
    out = _csa(O, d, m)
    for i in range(ne):
        rows = [d["Ca"][0, m * i:m * i + m]]
        if i > 0:
            rows.append(d["Cb"][0, m * (i - 1):m * i])
        V = np.vstack(rows)
        assert np.all(out[0, i] <= V.max(0) + 1e-15) and np.all(out[0, i] >= V.min(0) - 1e-15)


def pin_linearity_in_C(O):
    rng = np.random.default_rng(10)
    m = 4
    d1 = _rand_csa(rng, 1, 24, 5, m)
    d2 = dict(d1, Ca=rng.standard_normal(d1["Ca"].shape), Cb=rng.standard_normal(d1["Cb"].shape))
    dsum = dict(d1, Ca=2 * d1["Ca"] - 3 * d2["Ca"], Cb=2 * d1["Cb"] - 3 * d2["Cb"])
    assert np.allclose(_csa(O, dsum, m), 2 * _csa(O, d1, m) - 3 * _csa(O, d2, m), rtol=1e-12, atol=1e-12)


def pin_batch_independence(O):
    rng = np.random.default_rng(12)
    m = 4
    d = _rand_csa(rng, 3, 20, 4, m)
    full = _csa(O, d, m)
    for b in range(3):
        one = {k: (v[b:b + 1] if v.ndim == 3 else v) for k, v in d.items()}
        assert np.array_equal(_csa(O, one, m)[0], full[b])
    d2 = {k: v.copy() for k, v in d.items()}
    d2["Zb"][1] += 5.0
    d2["Cb"][1] -= 2.0
    out = _csa(O, d2, m)
    assert np.array_equal(out[0], full[0]) and np.array_equal(out[2], full[2])
    assert not np.array_equal(out[1, 1:], full[1, 1:])


def pin_tail_ignored(O):
    rng = np.random.default_rng(13)
    m = 4
    d = _rand_csa(rng, 1, 4 * 5 + 3, 4, m)
    base = _csa(O, d, m)
    assert base.shape[1] == 5
    d2 = {k: v.copy() for k, v in d.items()}
    for k in ("Ca", "Cb", "Za", "Zb"):
        d2[k][0, 20:] = 99.0
    assert np.array_equal(_csa(O, d2, m), base)


def pin_overlap_off(O):
    """overlap = False: each entry pools its own m rows of stream a only (the pages'
    non-overlapped grouping); a closed form against scipy + fsum."""
    rng = np.random.default_rng(14)
    m = 4
    d = _rand_csa(rng, 1, 16, 3, m)
    out = O.csa_compress(d["Ca"], None, d["Za"], None, d["Ba"], None, m, False)
    for i in range(4):
        assert np.allclose(out[0, i], _fsum_pool(d["Za"][0, 4 * i:4 * i + 4] + d["Ba"], d["Ca"][0, 4 * i:4 * i + 4]),
                           rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------------------------------
# Projection (fused path)
# --------------------------------------------------------------------------------------

def pin_projection_fsum(O):
    """H W against exactly rounded dot products, with d != c so a transposed operand
    cannot pass."""
    rng = np.random.default_rng(15)
    H = rng.standard_normal((5, 7))
    W = rng.standard_normal((7, 3))
    P = O.project(H, W)
    assert P.shape == (5, 3)
    for r in range(5):
        for ch in range(3):
            assert abs(P[r, ch] - math.fsum(H[r, k] * W[k, ch] for k in range(7))) < 1e-13


def pin_fused_stream_roles(O):
    """Scaled identities (d = c) make each stream a known multiple of H; the fused
    oracle must equal the streaming definition on those streams, which fixes which W
    feeds which stream."""
    rng = np.random.default_rng(16)
    m, n, c, batch = 4, 24, 6, 2
    H = rng.standard_normal((batch * n, c))
    I = np.eye(c)
    Ba, Bb = rng.standard_normal((m, c)), rng.standard_normal((m, c))
    out = O.csa_compress_fused(H, 1.0 * I, -2.0 * I, 0.5 * I, 3.0 * I, Ba, Bb, batch, n, m, True)
    Hs = H.reshape(batch, n, c)
    ref = O.csa_compress(1.0 * Hs, -2.0 * Hs, 0.5 * Hs, 3.0 * Hs, Ba, Bb, m, True)
    assert np.allclose(out, ref, rtol=1e-13, atol=1e-13)
    # and directly against the library-softmax evaluation for one interior entry
    i = 3
    La = 0.5 * Hs[1, 12:16] + Ba
    Lb = 3.0 * Hs[1, 8:12] + Bb
    refi = _fsum_pool(np.vstack([La, Lb]), np.vstack([Hs[1, 12:16], -2.0 * Hs[1, 8:12]]))
    assert np.allclose(out[1, i], refi, rtol=1e-13, atol=1e-13)
    # HCA
    B = rng.standard_normal((8, c))
    outh = O.hca_compress_fused(H, 2.0 * I, -1.0 * I, B, batch, n, 8)
    refh = O.hca_compress(2.0 * Hs, -1.0 * Hs, B, 8)
    assert np.allclose(outh, refh, rtol=1e-13, atol=1e-13)
    refh1 = _fsum_pool(-Hs[0, 8:16] + B, 2.0 * Hs[0, 8:16])
    assert np.allclose(outh[0, 1], refh1, rtol=1e-13, atol=1e-13)


def pin_fused_selection(O):
    """W that copies input feature perm[ch] to channel ch (d != c) makes the stream a
    column gather of H: fused == streaming on the gathered streams."""
    rng = np.random.default_rng(17)
    m, n, d, c = 4, 20, 9, 5
    H = rng.standard_normal((n, d))
    Ws, streams = [], []
    for s in range(4):
        perm = rng.choice(d, size=c, replace=False)
        W = np.zeros((d, c))
        W[perm, np.arange(c)] = 1.0
        Ws.append(W)
        streams.append(H[:, perm][None])
    Ba, Bb = rng.standard_normal((m, c)), rng.standard_normal((m, c))
    out = O.csa_compress_fused(H, Ws[0], Ws[1], Ws[2], Ws[3], Ba, Bb, 1, n, m, True)
    ref = O.csa_compress(streams[0], streams[1], streams[2], streams[3], Ba, Bb, m, True)
    assert np.allclose(out, ref, rtol=1e-13, atol=1e-13)
    ent = O.csa_compress_fused(H, Ws[0], Ws[1], Ws[2], Ws[3], Ba, Bb, 1, n, m, True,
                               entries=[(0, 4), (0, 0)])
    assert np.allclose(ent, ref[0, [4, 0]], rtol=1e-13, atol=1e-13)


# --------------------------------------------------------------------------------------
# Scalar-logit form ("Ch 04 · CSA" §3 symbol table: one score per token, S_j a scalar)
# --------------------------------------------------------------------------------------

def _rand_scalar(rng, batch, n, c, m):
    f = lambda *s: rng.standard_normal(s)
    return dict(Ca=f(batch, n, c), Cb=f(batch, n, c), za=2 * f(batch, n), zb=2 * f(batch, n),
                ba=0.3 * f(m), bb=0.3 * f(m))


def pin_scalar_is_channel_constant_case(O):
    """Scalar logits are the per-channel form with Z and B constant across channels (a
    special case of the pinned per-channel definition)."""
    rng = np.random.default_rng(31)
    m, c = 4, 5
    d = _rand_scalar(rng, 2, 4 * 7 + 2, c, m)
    out = O.csa_compress_scalar(d["Ca"], d["Cb"], d["za"], d["zb"], d["ba"], d["bb"], m, True)
    rep = lambda z: np.repeat(z[..., None], c, axis=-1)
    ref = O.csa_compress(d["Ca"], d["Cb"], rep(d["za"]), rep(d["zb"]), rep(d["ba"]), rep(d["bb"]), m, True)
    assert np.allclose(out, ref, rtol=1e-13, atol=1e-13)
    C = rng.standard_normal((1, 256, c))
    z = rng.standard_normal((1, 256)) * 3
    b = rng.standard_normal(128)
    assert np.allclose(O.hca_compress_scalar(C, z, b, 128), O.hca_compress(C, rep(z), rep(b), 128),
                       rtol=1e-13, atol=1e-13)


def pin_scalar_weights_via_unit_rows(O):
    """With the window's value rows set to unit vectors the entry IS the weight vector:
    it must equal scipy's softmax of [z^a + b^a; z^b + b^b] (entry 0: a-rows only)."""
    from scipy.special import softmax

    rng = np.random.default_rng(32)
    m, ne = 4, 5
    n = m * ne
    d = _rand_scalar(rng, 1, n, 2 * m, m)
    for i in range(ne):
        Ca = np.zeros((1, n, 2 * m))
        Cb = np.zeros((1, n, 2 * m))
        for k in range(m):
            Ca[0, m * i + k, k] = 1.0
            if i > 0:
                Cb[0, m * (i - 1) + k, m + k] = 1.0
        out = O.csa_compress_scalar(Ca, Cb, d["za"], d["zb"], d["ba"], d["bb"], m, True,
                                    entries=[(0, i)])[0]
        La = d["za"][0, m * i:m * i + m] + d["ba"]
        if i == 0:
            ref = np.concatenate([softmax(La), np.zeros(m)])
        else:
            ref = softmax(np.concatenate([La, d["zb"][0, m * (i - 1):m * i] + d["bb"]]))
        assert np.allclose(out, ref, rtol=1e-13, atol=1e-14), i


def pin_scalar_one_hot_and_logistic(O):
    rng = np.random.default_rng(33)
    m, ne, c = 4, 4, 3
    n = m * ne
    d = _rand_scalar(rng, 1, n, c, m)
    for r in range(n):
        for zs, cs, target in (("za", "Ca", r // m), ("zb", "Cb", r // m + 1)):
            if target >= ne:
                continue
            d2 = {k: v.copy() for k, v in d.items()}
            d2[zs][0, r] += 60.0
            out = O.csa_compress_scalar(d2["Ca"], d2["Cb"], d2["za"], d2["zb"], d2["ba"], d2["bb"], m,
                                        True, entries=[(0, target)])
            assert np.allclose(out[0], d[cs][0, r], rtol=1e-12, atol=1e-12), (zs, r)
    e = _rand_scalar(rng, 1, 7, c, 1)
    out = O.csa_compress_scalar(e["Ca"], e["Cb"], e["za"], e["zb"], e["ba"], e["bb"], 1, True)
    for i in range(1, 7):
        x = e["za"][0, i] + e["ba"][0] - e["zb"][0, i - 1] - e["bb"][0]
        s = 1.0 / (1.0 + math.exp(-x))
        assert np.allclose(out[0, i], s * e["Ca"][0, i] + (1 - s) * e["Cb"][0, i - 1], rtol=1e-13, atol=1e-13)
    assert np.allclose(out[0, 0], e["Ca"][0, 0], rtol=0, atol=1e-15)
    # HCA: bias one-hot selects in-segment position k
    C = rng.standard_normal((1, 256, c))
    z = rng.standard_normal((1, 256))
    b = np.zeros(128)
    b[77] = 60.0
    out = O.hca_compress_scalar(C, z, b, 128)
    assert np.allclose(out[0, 1], C[0, 128 + 77], rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------------------
# Cache-format epilogue: FP8 E4M3 rounding and pair-wise RoPE
# --------------------------------------------------------------------------------------

def _e4m3_codes():
    """All finite non-negative E4M3 values decoded from the bit fields of the format
    (4 exponent bits with bias 7, 3 mantissa bits; exponent field 0 is subnormal;
    exponent 15 with mantissa 7 is NaN), in code order."""
    vals = []
    for e in range(16):
        for mm in range(8):
            if e == 15 and mm == 7:
                continue
            vals.append(mm / 8 * 2.0 ** -6 if e == 0 else (1 + mm / 8) * 2.0 ** (e - 7))
    return np.array(vals)


def pin_e4m3_rounding(O):
    v = _e4m3_codes()
    assert v[-1] == 448.0 and v[1] == 2.0 ** -9
    assert np.array_equal(O.round_e4m3(v), v) and np.array_equal(O.round_e4m3(-v), -v)
    mids = (v[:-1] + v[1:]) / 2
    got = O.round_e4m3(mids)
    for k, g in enumerate(got):       # ties go to the even code
        assert g == (v[k] if k % 2 == 0 else v[k + 1]), (k, mids[k], g)
    inside = (v[:-1] + 0.49 * (v[1:] - v[:-1]))
    assert np.array_equal(O.round_e4m3(inside), v[:-1])
    assert np.all(O.round_e4m3(np.array([449.0, 1e6, -5e3])) == np.array([448.0, 448.0, -448.0]))
    import torch  # library cast (saturation excluded: torch maps overflow to NaN)
    x = np.random.default_rng(40).standard_normal(20000) * 40
    x = np.clip(x, -448, 448)
    t = torch.from_numpy(x).to(torch.float8_e4m3fn).double().numpy()
    assert np.array_equal(O.round_e4m3(x), t)


def pin_rope_closed_forms(O):
    rng = np.random.default_rng(41)
    r = 8
    inv = 10000.0 ** (-np.arange(r // 2) * 2 / r)
    x = rng.standard_normal((5, r))
    assert np.allclose(O.rope_pairs(x, np.zeros(5), inv), x, rtol=0, atol=1e-15)
    pos = rng.uniform(0, 5000, 5)
    y = O.rope_pairs(x, pos, inv)
    for t in range(5):
        for j in range(r // 2):
            a = pos[t] * inv[j]
            ref = (x[t, 2 * j] * math.cos(a) - x[t, 2 * j + 1] * math.sin(a),
                   x[t, 2 * j] * math.sin(a) + x[t, 2 * j + 1] * math.cos(a))
            assert abs(y[t, 2 * j] - ref[0]) < 1e-12 and abs(y[t, 2 * j + 1] - ref[1]) < 1e-12
    p2 = rng.uniform(0, 100, 5)
    assert np.allclose(O.rope_pairs(y, p2, inv), O.rope_pairs(x, pos + p2, inv), rtol=1e-10, atol=1e-10)


def pin_cache_format_layout(O):
    rng = np.random.default_rng(42)
    e = rng.standard_normal((2, 6, 24)) * 3
    r = 8
    inv = rng.uniform(0, 1, r // 2)
    nope, rope = O.cache_format(e, r, inv, pos_stride=4.0, pos_offset=1.5, scale=2.0)
    assert nope.shape == (2, 6, 16) and rope.shape == (2, 6, 8)
    assert np.array_equal(nope, O.round_e4m3(e[..., :16] * 2.0))
    for i in range(6):
        a = (1.5 + 4.0 * i) * inv[1]
        assert abs(rope[1, i, 2] - (e[1, i, 18] * math.cos(a) - e[1, i, 19] * math.sin(a))) < 1e-12


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
