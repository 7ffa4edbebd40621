"""fp64 CPU oracle of the token-level KV compressor (CSA overlap / HCA).

TEST INFRASTRUCTURE. Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s
cpu_baseline / reference legs may import or run this module.  The product package
(``kv_token_compressor_b200``) never imports it and shares no code with it.

It is the plain definition of the method, written out step by step in float64 with
numpy (no blocking, fusion or reordering beyond what the equations state):

* Streams (page "序列压缩注意力", section "compressor 怎么把多个 token 压成一个 KV entry",
  eq. attn-seqcomp-csa-proj):  C^a = H W^{KV_a}, C^b = H W^{KV_b}, Z^a = H W^{Z_a},
  Z^b = H W^{Z_b}, each n x c.
* CSA entry i (same section, eq. attn-seqcomp-csa-softmax and eq. attn-seqcomp-csa-pool;
  also "Ch 04 · CSA", §3 Token-Level Compressor): stack the 2m logit rows
  [Z^a_{mi..m(i+1)-1} + B^a ; Z^b_{m(i-1)..mi-1} + B^b], softmax each channel jointly
  over those 2m rows, and pool C^Comp_i = sum S^a (.) C^a + sum S^b (.) C^b.
* Coverage (same page, section "overlap transform …", table attn-seqcomp-overlap):
  a-range(i) = [mi, m(i+1)-1], b-range(i) = [m(i-1), mi-1].
* Entry 0 (same section, eq. attn-seqcomp-overlap-bound): the missing b-rows at
  positions -m..-1 get logit -inf and vector 0.  They are padded here literally.
* HCA (same page, section "HCA 怎么靠 128× 压缩做 dense attention", eq. attn-seqcomp-hca;
  "Ch 05 · HCA", §2 compression formulas): S = Softmax_row(Z + B) over the m' rows of
  segment i, C^Comp_i = sum S_j (.) C_j, no overlap, single stream.

Readings taken where the pages are silent or disagree:
Z and B are per channel (n x c and m x c), the softmax is joint over the 2m rows, the
entry count is floor(n/m) with the trailing n mod m tokens not compressed, sequences of
a batch are independent, the fused path keeps the streams unrounded (float64 here).

All array arguments may be any real dtype; they are widened exactly to float64
(bf16 and fp32 values are exactly representable in float64).
"""

from __future__ import annotations

import numpy as np

__all__ = [
    "num_entries",
    "entry_rows",
    "softmax_rows",
    "pool_window",
    "csa_window",
    "csa_entry",
    "csa_compress",
    "hca_entry",
    "hca_compress",
    "project",
    "csa_compress_fused",
    "hca_compress_fused",
    "csa_entry_scalar",
    "csa_compress_scalar",
    "hca_entry_scalar",
    "hca_compress_scalar",
    "round_e4m3",
    "rope_pairs",
    "cache_format",
]


def _f64(x):
    return np.asarray(x, dtype=np.float64)


def num_entries(n: int, m: int) -> int:
    """Number of compressed entries of an n-token sequence at ratio m.

    "Ch 04 · CSA", §3 (naive compression cuts the sequence into floor(n/m) segments);
    "序列压缩注意力", table attn-seqcomp-csa-hca (n tokens -> about n/m entries).
    The trailing n mod m tokens form no complete block and are not compressed.
    """
    if m <= 0:
        raise ValueError("m must be positive")
    if n < 0:
        raise ValueError("n must be non-negative")
    return n // m


def entry_rows(i: int, m: int):
    """Token rows read by CSA entry i: (a-range, b-range) as Python ranges.

    "序列压缩注意力", table attn-seqcomp-overlap: stream C^a covers [mi, m(i+1)-1],
    stream C^b covers [m(i-1), mi-1].  For i = 0 the b-range is [-m, -1], positions
    that do not exist (eq. attn-seqcomp-overlap-bound).
    """
    return range(m * i, m * (i + 1)), range(m * (i - 1), m * i)


def softmax_rows(L):
    """Softmax of every column of L taken over its rows ("Softmax_row" of the pages).

    S[k, ch] = exp(L[k, ch] - M[ch]) / sum_k' exp(L[k', ch] - M[ch]) with
    M[ch] = max_k L[k, ch].  Subtracting M changes nothing mathematically; rows at -inf
    get weight exactly 0.
    """
    L = _f64(L)
    M = np.max(L, axis=0, keepdims=True)
    w = np.exp(L - M)
    return w / np.sum(w, axis=0, keepdims=True)


def pool_window(L, V):
    """sum_k S[k] (.) V[k] with S = softmax_rows(L): one compressed entry.

    L and V are (rows, c).  This is eq. attn-seqcomp-csa-pool / attn-seqcomp-hca of
    "序列压缩注意力" for the rows of one window.
    """
    S = softmax_rows(L)
    return np.sum(S * _f64(V), axis=0)


def csa_window(Ca, Cb, Za, Zb, Ba, Bb, i: int, m: int, overlap: bool = True):
    """The logit rows and value rows of CSA entry i of ONE sequence ([n, c] streams).

    Returns (L, V), each (2m, c) with overlap (a-rows first, then b-rows), or (m, c)
    without.  Entry 0's b-rows are the boundary rows: logit -inf, vector 0.
    Bias row k pairs with in-block position k of its block (eq.
    attn-seqcomp-csa-softmax adds B^a to Z^a_{mi..m(i+1)-1}, B^b to Z^b_{m(i-1)..mi-1}).
    """
    a_rows, b_rows = entry_rows(i, m)
    c = np.shape(Ca)[1]
    La = _f64(Za[a_rows.start:a_rows.stop]) + _f64(Ba)
    Va = _f64(Ca[a_rows.start:a_rows.stop])
    if not overlap:
        return La, Va
    Bb = _f64(Bb)
    if i == 0:
        Zb_rows = np.full((m, c), -np.inf)   # Z^b_{-m:-1} = -inf
        Cb_rows = np.zeros((m, c))           # C^b_{-m:-1} = 0
    else:
        Zb_rows = _f64(Zb[b_rows.start:b_rows.stop])
        Cb_rows = _f64(Cb[b_rows.start:b_rows.stop])
    Lb = Zb_rows + Bb
    L = np.concatenate([La, Lb], axis=0)
    V = np.concatenate([Va, Cb_rows], axis=0)
    return L, V


def csa_entry(Ca, Cb, Za, Zb, Ba, Bb, i: int, m: int, overlap: bool = True):
    """C^Comp_i of one sequence (eqs. attn-seqcomp-csa-softmax / -csa-pool)."""
    L, V = csa_window(Ca, Cb, Za, Zb, Ba, Bb, i, m, overlap)
    return pool_window(L, V)


def _entry_list(batch: int, ne: int, entries):
    if entries is None:
        return [(b, i) for b in range(batch) for i in range(ne)]
    out = []
    for b, i in entries:
        if not (0 <= b < batch and 0 <= i < ne):
            raise IndexError(f"entry ({b}, {i}) out of range")
        out.append((int(b), int(i)))
    return out


def csa_compress(Ca, Cb, Za, Zb, Ba, Bb, m: int = 4, overlap: bool = True, entries=None):
    """CSA compressor over a batch of sequences.

    Streams are [batch, n, c]; Ba, Bb are [m, c] (Cb, Zb, Bb may be None when
    overlap is False).  Returns float64 [batch, floor(n/m), c], or, when ``entries``
    lists (b, i) pairs, float64 [len(entries), c] with just those entries.
    Sequences are independent: no window crosses a sequence boundary.
    """
    batch, n, c = np.shape(Ca)
    ne = num_entries(n, m)
    todo = _entry_list(batch, ne, entries)
    rows = []
    for b, i in todo:
        Cb_b = None if Cb is None else Cb[b]
        Zb_b = None if Zb is None else Zb[b]
        rows.append(csa_entry(Ca[b], Cb_b, Za[b], Zb_b, Ba, Bb, i, m, overlap))
    res = np.array(rows, dtype=np.float64).reshape(len(todo), c)
    if entries is None:
        return res.reshape(batch, ne, c)
    return res


def hca_entry(C, Z, B, i: int, m: int):
    """C^Comp_i of one sequence for HCA (eq. attn-seqcomp-hca): softmax of Z + B over
    the m rows of segment i = [m i, m(i+1)-1], then the weighted sum of those C rows."""
    lo, hi = m * i, m * (i + 1)
    L = _f64(Z[lo:hi]) + _f64(B)
    return pool_window(L, _f64(C[lo:hi]))


def hca_compress(C, Z, B, m: int = 128, entries=None):
    """HCA compressor over [batch, n, c] streams with bias B [m, c].  Output as in
    :func:`csa_compress`."""
    batch, n, c = np.shape(C)
    ne = num_entries(n, m)
    todo = _entry_list(batch, ne, entries)
    rows = [hca_entry(C[b], Z[b], B, i, m) for b, i in todo]
    res = np.array(rows, dtype=np.float64).reshape(len(todo), c)
    if entries is None:
        return res.reshape(batch, ne, c)
    return res


def project(H, W):
    """H W in float64 (eq. attn-seqcomp-csa-proj): H is [rows, d], W is [d, c]."""
    return _f64(H) @ _f64(W)


def _check_fused_shapes(H, W, batch, n):
    if np.ndim(H) != 2 or np.shape(H)[0] != batch * n:
        raise ValueError("H must be [batch*n, d]")
    if np.asarray(W).shape[0] != H.shape[1]:
        raise ValueError("W must be [d, c]")


def csa_compress_fused(H, W_kva, W_kvb, W_za, W_zb, Ba, Bb, batch: int, n: int,
                       m: int = 4, overlap: bool = True, entries=None):
    """CSA compressor fed by hidden states: the streams are H W (float64, never
    rounded), then pooled exactly as :func:`csa_compress`.

    H is [batch*n, d] (sequence b occupies rows b*n .. b*n+n-1); each W is [d, c].
    Only the token rows that the requested entries read are projected.
    """
    _check_fused_shapes(H, W_kva, batch, n)
    c = np.asarray(W_kva).shape[1]
    ne = num_entries(n, m)
    todo = _entry_list(batch, ne, entries)
    out = np.empty((len(todo), c))
    for t, (b, i) in enumerate(todo):
        a_rows, b_rows = entry_rows(i, m)
        lo = m * (i - 1) if (overlap and i > 0) else m * i
        hi = m * (i + 1)
        Hs = _f64(H[b * n + lo:b * n + hi])      # the tokens entry i reads
        # Place the projected rows at their token positions of a local [hi, c] view.
        def stream(W):
            S = np.zeros((hi, c))
            S[lo:hi] = project(Hs, W)
            return S
        Ca, Za = stream(W_kva), stream(W_za)
        Cb = stream(W_kvb) if overlap else None
        Zb = stream(W_zb) if overlap else None
        out[t] = csa_entry(Ca, Cb, Za, Zb, Ba, Bb, i, m, overlap)
    if entries is None:
        return out.reshape(batch, ne, c)
    return out


def hca_compress_fused(H, W_kv, W_z, B, batch: int, n: int, m: int = 128, entries=None):
    """HCA compressor fed by hidden states: C = H W^{KV}, Z = H W^{Z} in float64 for
    the m rows of each requested segment, then :func:`hca_entry`."""
    _check_fused_shapes(H, W_kv, batch, n)
    c = np.asarray(W_kv).shape[1]
    ne = num_entries(n, m)
    todo = _entry_list(batch, ne, entries)
    out = np.empty((len(todo), c))
    for t, (b, i) in enumerate(todo):
        Hs = _f64(H[b * n + m * i:b * n + m * (i + 1)])
        C = project(Hs, W_kv)
        Z = project(Hs, W_z)
        out[t] = hca_entry(C, Z, B, 0, m)
    if entries is None:
        return out.reshape(batch, ne, c)
    return out


# --------------------------------------------------------------------------------------
# Scalar-logit form.  "Ch 04 · CSA" §3's symbol table reads the same equations with one
# score per token and stream (Z^a, Z^b of dimension n), an m-dimensional bias B^a, B^b,
# and S_j a scalar that multiplies the whole vector C_j; "Ch 05 · HCA" §2 likewise gives
# B as m'-dimensional.  The softmax is still joint over the window's rows.
# --------------------------------------------------------------------------------------

def csa_entry_scalar(Ca, Cb, za, zb, ba, bb, i: int, m: int, overlap: bool = True):
    """C^Comp_i of one sequence with scalar logits: za, zb are [n], ba, bb are [m]."""
    a_rows, b_rows = entry_rows(i, m)
    la = _f64(za[a_rows.start:a_rows.stop]) + _f64(ba)
    va = _f64(Ca[a_rows.start:a_rows.stop])
    if overlap:
        if i == 0:
            lb = np.full(m, -np.inf)                 # Z^b_{-m:-1} = -inf
            vb = np.zeros((m, np.shape(Ca)[1]))      # C^b_{-m:-1} = 0
        else:
            lb = _f64(zb[b_rows.start:b_rows.stop]) + _f64(bb)
            vb = _f64(Cb[b_rows.start:b_rows.stop])
        L = np.concatenate([la, lb])
        V = np.concatenate([va, vb], axis=0)
    else:
        L, V = la, va
    w = np.exp(L - np.max(L))
    s = w / np.sum(w)                                # one weight per row, shared by channels
    return np.sum(s[:, None] * V, axis=0)


def csa_compress_scalar(Ca, Cb, za, zb, ba, bb, m: int = 4, overlap: bool = True, entries=None):
    """CSA compressor with scalar logits.  Ca, Cb: [batch, n, c]; za, zb: [batch, n];
    ba, bb: [m].  Output as in :func:`csa_compress`."""
    batch, n, c = np.shape(Ca)
    ne = num_entries(n, m)
    todo = _entry_list(batch, ne, entries)
    rows = [csa_entry_scalar(Ca[b], None if Cb is None else Cb[b], za[b],
                             None if zb is None else zb[b], ba, bb, i, m, overlap)
            for b, i in todo]
    res = np.array(rows, dtype=np.float64).reshape(len(todo), c)
    return res.reshape(batch, ne, c) if entries is None else res


def hca_entry_scalar(C, z, bvec, i: int, m: int):
    """HCA segment i with scalar logits z [n] and bias bvec [m]."""
    lo, hi = m * i, m * (i + 1)
    L = _f64(z[lo:hi]) + _f64(bvec)
    w = np.exp(L - np.max(L))
    s = w / np.sum(w)
    return np.sum(s[:, None] * _f64(C[lo:hi]), axis=0)


def hca_compress_scalar(C, z, bvec, m: int = 128, entries=None):
    """HCA compressor with scalar logits: C [batch, n, c], z [batch, n], bvec [m]."""
    batch, n, c = np.shape(C)
    ne = num_entries(n, m)
    todo = _entry_list(batch, ne, entries)
    rows = [hca_entry_scalar(C[b], z[b], bvec, i, m) for b, i in todo]
    res = np.array(rows, dtype=np.float64).reshape(len(todo), c)
    return res.reshape(batch, ne, c) if entries is None else res


# --------------------------------------------------------------------------------------
# Cache-format epilogue.  "Ch 05 · HCA" §4 (2): RoPE acts on the last r = 64 dimensions
# of each entry only, rotating adjacent pairs of dimensions by a position-dependent angle,
# the other c - r stay position-free; the segment position is carried approximately by
# the rope dimensions (segment-centre RoPE).  The CSA/HCA comparison article (section
# 三.4, mixed-precision storage) stores the RoPE part in BF16 and the other KV values in
# FP8.  Readings (the pages fix neither): the caller supplies the inverse frequencies of
# the r/2 pairs and the entry position pos_i = pos_offset + pos_stride * i; FP8 is
# E4M3 (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no infinities, largest
# finite 448), round to nearest even, saturating, after multiplying by a caller scale.
# --------------------------------------------------------------------------------------

E4M3_MAX = 448.0


def round_e4m3(x):
    """Nearest FP8 E4M3 value (ties to even), saturating to +-448, as float64."""
    x = _f64(x)
    a = np.abs(x)
    mant, expo = np.frexp(a)                 # a = mant * 2^expo, mant in [0.5, 1)
    lead = expo - 1                          # exponent of the leading bit
    quantum = np.ldexp(1.0, np.maximum(lead, -6) - 3)   # 3 mantissa bits; subnormal step 2^-9
    q = np.round(a / quantum) * quantum      # numpy rounds half to even
    q = np.minimum(q, E4M3_MAX)
    return np.where(a == 0, 0.0, np.copysign(q, x))


def rope_pairs(x, pos, inv_freq):
    """Rotate adjacent pairs (2j, 2j+1) of x [..., r] by angle pos * inv_freq[j]."""
    x = _f64(x)
    r = x.shape[-1]
    ang = np.multiply.outer(_f64(pos), _f64(inv_freq))          # [..., r/2]
    z = (x[..., 0::2] + 1j * x[..., 1::2]) * np.exp(1j * ang)  # one complex number per pair
    out = np.empty_like(x)
    out[..., 0::2] = z.real
    out[..., 1::2] = z.imag
    assert out.shape[-1] == r
    return out


def cache_format(entries, r: int, inv_freq, pos_stride: float, pos_offset: float,
                 scale: float = 1.0):
    """Split compressed entries [batch, N_e, c] into the cache layout: the first c - r
    dimensions times `scale` rounded to E4M3, and the last r dimensions rotated at
    pos_i = pos_offset + pos_stride * i (i = entry index in its sequence), float64."""
    entries = _f64(entries)
    c = entries.shape[-1]
    ne = entries.shape[-2]
    pos = pos_offset + pos_stride * np.arange(ne, dtype=np.float64)
    pos = np.broadcast_to(pos, entries.shape[:-1])
    nope = round_e4m3(entries[..., :c - r] * scale)
    rope = rope_pairs(entries[..., c - r:], pos, inv_freq)
    return nope, rope
