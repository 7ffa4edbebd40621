"""GPU parity of the cache-layout epilogue (partial RoPE on the last r dimensions in bf16,
the rest scaled and rounded to FP8 E4M3) against the oracle's cache_format.

FP8 comparison: the kernel rounds its fp32 entry, the oracle its fp64 entry, so a value
lying within fp32 rounding of an E4M3 rounding boundary may land one code apart; every
code must be within one E4M3 step of the oracle's and almost all must be equal."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from gpu_util import check_close, dev, host64
from kv_token_compressor_b200 import kvc, synth
from oracle import compressor as O

pytestmark = pytest.mark.gpu


def _inv_freq(r, base=10000.0):
    return (base ** (-np.arange(r // 2, dtype=np.float64) * 2 / r)).astype(np.float32)


def _fp8_values(t):
    return t.contiguous().view(torch.float8_e4m3fn).to(torch.float64).cpu().numpy()


def _check_fp8(got, ref, what):
    got = np.asarray(got).reshape(ref.shape)
    step = np.maximum(2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -6))) - 3), 2.0 ** -9)
    assert np.all(np.abs(got - ref) <= step * 1.0001), f"{what}: fp8 code beyond one step"
    frac = np.mean(got != ref) if ref.size else 0.0
    assert frac <= 2e-3, f"{what}: {frac:.4%} of fp8 codes differ"


def _compare(nope, rope, entries64, r, inv, stride, offset, scale, what):
    ref_nope, ref_rope = O.cache_format(entries64, r, inv.astype(np.float64), stride, offset, scale)
    if ref_nope.size:
        _check_fp8(_fp8_values(nope), ref_nope, what + " nope")
    if ref_rope.size:
        check_close(rope, ref_rope, "bf16", what + " rope")


@pytest.mark.parametrize("dt", ["bf16", "f32"])
@pytest.mark.parametrize("r", [64, 0, 512])
def test_csa_cache(dt, r):
    batch, n, c, m = 2, 4 * 100 + 3, 512, 4
    d = synth.stream_inputs("csa", batch, n, c, m, dt, seed=r + (dt == "f32"))
    t = {k: dev(v, dt) if v.ndim == 3 else dev(v, "f32") for k, v in d.items()}
    inv = _inv_freq(max(r, 2))
    nope, rope = kvc.csa_compress_cache(t["Ca"], t["Cb"], t["Za"], t["Zb"], t["Ba"], t["Bb"], r,
                                        torch.from_numpy(inv).cuda(), pos_stride=4.0,
                                        pos_offset=1.5, fp8_scale=2.0, m=m)
    torch.cuda.synchronize()
    ref = O.csa_compress(d["Ca"], d["Cb"], d["Za"], d["Zb"], d["Ba"], d["Bb"], m, True)
    _compare(nope, rope, ref, r, inv[:r // 2], 4.0, 1.5, 2.0, f"csa cache r={r} {dt}")


def test_hca_cache_large_positions_and_saturation():
    batch, n, c, m, r = 1, 128 * 12, 512, 128, 64
    d = synth.stream_inputs("hca", batch, n, c, m, "bf16", seed=7)
    t = {k: dev(v, "bf16") if v.ndim == 3 else dev(v, "f32") for k, v in d.items()}
    inv = _inv_freq(r)
    # positions near 2^20 exercise the fp64 range reduction; scale 2000 saturates many codes
    nope, rope = kvc.hca_compress_cache(t["C"], t["Z"], t["B"], r, torch.from_numpy(inv).cuda(),
                                        pos_stride=128.0, pos_offset=1048000.5, fp8_scale=2000.0)
    torch.cuda.synchronize()
    ref = O.hca_compress(d["C"], d["Z"], d["B"], m)
    _compare(nope, rope, ref, r, inv, 128.0, 1048000.5, 2000.0, "hca cache")
    assert np.any(np.abs(_fp8_values(nope)) == 448.0)


def test_listed_cache_insertion():
    """Decode: each sequence's newest entry goes straight into the cache layout, at its
    own position in its sequence."""
    m, c, r = 4, 512, 64
    rng = np.random.default_rng(3)
    lens = [int(x) for x in rng.integers(8, 2000, size=19)]
    d = synth.stream_inputs("csa", 1, sum(lens), c, m, "bf16", seed=3)
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]])
    ents = [(s, L // m - 1) for s, L in enumerate(lens)]
    t = {k: dev(v[0], "bf16") if v.ndim == 3 else dev(v, "f32") for k, v in d.items()}
    idx = lambda xs: torch.tensor(xs, dtype=torch.int64, device="cuda")
    inv = _inv_freq(r)
    nope, rope = kvc.csa_compress_entries_cache(
        t["Ca"], t["Cb"], t["Za"], t["Zb"], t["Ba"], t["Bb"], idx([starts[s] for s, _ in ents]),
        idx([lens[s] for s, _ in ents]), idx([e for _, e in ents]), r, torch.from_numpy(inv).cuda(),
        pos_stride=4.0, pos_offset=1.5, fp8_scale=1.0)
    torch.cuda.synchronize()
    assert kvc.device_status() == kvc.KVC_OK
    refs, poss = [], []
    for s, e in ents:
        sl = slice(starts[s], starts[s] + lens[s])
        refs.append(O.csa_compress(d["Ca"][:, sl], d["Cb"][:, sl], d["Za"][:, sl], d["Zb"][:, sl],
                                   d["Ba"], d["Bb"], m, True, entries=[(0, e)])[0])
        poss.append(1.5 + 4.0 * e)
    ent = np.array(refs)
    ref_nope = O.round_e4m3(ent[:, :c - r])
    ref_rope = O.rope_pairs(ent[:, c - r:], np.array(poss), inv.astype(np.float64))
    _check_fp8(_fp8_values(nope), ref_nope, "listed nope")
    check_close(rope, ref_rope, "bf16", "listed rope")


@pytest.mark.parametrize("dt", ["bf16", "f32"])
def test_hca_listed_cache_insertion(dt):
    """HCA decode: each sequence's newest complete 128-row entry, in a shuffled list, goes
    into the cache layout at its own position in its sequence."""
    m, c, r = 128, 256, 64
    rng = np.random.default_rng(11)
    lens = [int(x) for x in rng.integers(m, 12 * m, size=9)]
    d = synth.stream_inputs("hca", 1, sum(lens), c, m, dt, seed=12)
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]])
    ents = [(s, L // m - 1) for s, L in enumerate(lens)]
    rng.shuffle(ents)
    t = {k: dev(v[0], dt) if v.ndim == 3 else dev(v, "f32") for k, v in d.items()}
    idx = lambda xs: torch.tensor([int(x) for x in xs], dtype=torch.int64, device="cuda")
    inv = _inv_freq(r)
    stride, offset = 128.0, 63.5
    nope, rope = kvc.hca_compress_entries_cache(
        t["C"], t["Z"], t["B"], idx([starts[s] for s, _ in ents]), idx([lens[s] for s, _ in ents]),
        idx([e for _, e in ents]), r, torch.from_numpy(inv).cuda(), pos_stride=stride,
        pos_offset=offset, fp8_scale=1.5)
    torch.cuda.synchronize()
    assert kvc.device_status() == kvc.KVC_OK
    refs, poss = [], []
    for s, e in ents:
        sl = slice(starts[s], starts[s] + lens[s])
        refs.append(O.hca_compress(d["C"][:, sl], d["Z"][:, sl], d["B"], m)[0, e])
        poss.append(offset + stride * e)
    ent = np.array(refs)
    ref_nope = O.round_e4m3(ent[:, :c - r] * 1.5)
    ref_rope = O.rope_pairs(ent[:, c - r:], np.array(poss), inv.astype(np.float64))
    _check_fp8(_fp8_values(nope), ref_nope, "hca listed nope")
    check_close(rope, ref_rope, "bf16", "hca listed rope")


@pytest.mark.parametrize("seed", range(4))
def test_cache_random_layouts(seed):
    """Seeded random cache layouts: c a multiple of 8, r a multiple of 8 in [0, c] (the
    layout's rule), position offset and stride, FP8 scale; CSA (m = 4) and HCA (m = 64 or
    128), bf16 or fp32 streams."""
    rng = np.random.default_rng(40 + seed)
    for mode in ("csa", "hca"):
        c = 8 * int(rng.integers(2, 97))
        r = 8 * int(rng.integers(0, c // 8 + 1))
        dt = rng.choice(["bf16", "f32"])
        m = 4 if mode == "csa" else int(rng.choice([64, 128]))
        batch, n = int(rng.integers(1, 3)), int(rng.integers(m, 30 * m))
        stride, offset = float(rng.choice([1.0, 4.0, 128.0])), float(rng.uniform(0, 5000))
        scale = float(rng.choice([0.5, 1.0, 8.0]))
        inv = _inv_freq(max(r, 2))
        d = synth.stream_inputs(mode, batch, n, c, m, dt, seed=seed * 5 + c)
        t = {k: dev(v, dt) if v.ndim == 3 else dev(v, "f32") for k, v in d.items()}
        invt = torch.from_numpy(inv).cuda()
        if mode == "csa":
            nope, rope = kvc.csa_compress_cache(t["Ca"], t["Cb"], t["Za"], t["Zb"], t["Ba"], t["Bb"], r,
                                                invt, pos_stride=stride, pos_offset=offset,
                                                fp8_scale=scale, m=m)
            ref = O.csa_compress(d["Ca"], d["Cb"], d["Za"], d["Zb"], d["Ba"], d["Bb"], m, True)
        else:
            nope, rope = kvc.hca_compress_cache(t["C"], t["Z"], t["B"], r, invt, pos_stride=stride,
                                                pos_offset=offset, fp8_scale=scale, m=m)
            ref = O.hca_compress(d["C"], d["Z"], d["B"], m)
        torch.cuda.synchronize()
        what = f"{mode} cache c={c} r={r} m={m} {dt} ({kvc.last_kernel()})"
        assert kvc.device_status() == kvc.KVC_OK, what
        _compare(nope, rope, ref, r, inv[:r // 2], stride, offset, scale, what)


def test_cache_rejects_bad_layout():
    x = torch.zeros((1, 64, 128), device="cuda", dtype=torch.bfloat16)
    b = torch.zeros((4, 128), device="cuda")
    inv = torch.ones(8, device="cuda")
    with pytest.raises(kvc.KvcError) as e:
        kvc.csa_compress_cache(x, x, x, x, b, b, 12, inv)   # r not a multiple of 8
    assert e.value.status == kvc.KVC_ERR_SHAPE
    with pytest.raises(kvc.KvcError) as e:
        kvc.csa_compress_cache(x, x, x, x, b, b, 136, inv)  # r > c
    assert e.value.status == kvc.KVC_ERR_SHAPE
