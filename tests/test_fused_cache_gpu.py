"""GPU parity of the fused compressors writing the cache layout straight from the GEMM
epilogue (csa/hca_compress_fused_proj_cache): the oracle's fused entries, put through its
cache_format (E4M3 for the first c - r dimensions after the scale, RoPE'd bf16 for the
last r), against the kernel's bytes.

FP8 comparison as in the streaming cache tests: the kernel rounds its fp32 entry and the
oracle its fp64 entry, so a value within fp32 rounding of an E4M3 boundary may land one
code apart; every code must be within one E4M3 step and almost all must be equal."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from gpu_util import check_close, host64
from kv_token_compressor_b200 import kvc, synth
from oracle import compressor as O

pytestmark = pytest.mark.gpu

GUARD = 256  # bytes of canary on each side of the E4M3 output (keeps it 16-byte aligned)


def _inv_freq(r, base=10000.0):
    return (base ** (-np.arange(max(r, 2) // 2, dtype=np.float64) * 2 / max(r, 2))).astype(np.float32)


def _fp8_values(t):
    return t.contiguous().view(torch.float8_e4m3fn).to(torch.float64).cpu().numpy()


def _check_fp8(got, ref, what):
    got = np.asarray(got).reshape(ref.shape)
    step = np.maximum(2.0 ** (np.floor(np.log2(np.maximum(np.abs(ref), 2.0 ** -6))) - 3), 2.0 ** -9)
    assert np.all(np.abs(got - ref) <= step * 1.0001), f"{what}: fp8 code beyond one step"
    frac = np.mean(got != ref) if ref.size else 0.0
    assert frac <= 2e-3, f"{what}: {frac:.4%} of fp8 codes differ"


def _dev(h):
    return {k: torch.from_numpy(np.ascontiguousarray(v)).cuda().to(
        torch.float32 if k.startswith("B") else torch.bfloat16) for k, v in h.items()}


def _guarded_cache_outs(rows, c, r):
    nb = torch.full((rows * (c - r) + 2 * GUARD,), 0x5A, dtype=torch.uint8, device="cuda")
    rb = torch.full((rows * r + 2 * GUARD,), -1280.0, dtype=torch.bfloat16, device="cuda")
    nope = nb[GUARD:GUARD + rows * (c - r)]
    rope = rb[GUARD:GUARD + rows * r]
    return nb, rb, nope, rope


def _guards_ok(nb, rb, rows, c, r):
    n_out, r_out = rows * (c - r), rows * r
    assert bool(torch.all(nb[:GUARD] == 0x5A)) and bool(torch.all(nb[GUARD + n_out:] == 0x5A))
    assert bool(torch.all(rb[:GUARD] == -1280.0)) and bool(torch.all(rb[GUARD + r_out:] == -1280.0))


def _compare(nope, rope, entries, r, inv, stride, offset, scale, what):
    ref_nope, ref_rope = O.cache_format(entries, r, inv[:r // 2].astype(np.float64), stride, offset,
                                        scale)
    if ref_nope.size:
        _check_fp8(_fp8_values(nope), ref_nope, what + " nope")
    if ref_rope.size:
        check_close(rope, ref_rope, "bf16", what + " rope")


@pytest.mark.parametrize("r", [64, 0, 512, 8])
def test_csa_fused_cache(r):
    batch, n, d, c = 2, 4 * 700 + 2, 128, 512
    h = synth.fused_inputs("csa", batch, n, d, c, 4, seed=r + 1)
    t = _dev(h)
    inv = _inv_freq(r)
    ne = n // 4
    nb, rb, nope, rope = _guarded_cache_outs(batch * ne, c, r)
    kvc.csa_compress_fused_proj_cache(t["H"], t["W_kva"], t["W_kvb"], t["W_za"], t["W_zb"], t["Ba"],
                                      t["Bb"], batch, n, r, torch.from_numpy(inv).cuda(),
                                      pos_stride=4.0, pos_offset=1.5, fp8_scale=2.0, out_nope=nope,
                                      out_rope=rope)
    assert kvc.last_kernel() == "fused_pair_kernel/csa/cache"
    assert kvc.device_status() == kvc.KVC_OK
    ent = O.csa_compress_fused(h["H"], h["W_kva"], h["W_kvb"], h["W_za"], h["W_zb"], h["Ba"],
                               h["Bb"], batch, n, 4, True)
    _compare(nope.view(batch, ne, c - r), rope.view(batch, ne, r), ent, r, inv, 4.0, 1.5, 2.0,
             f"csa fused cache r={r}")
    _guards_ok(nb, rb, batch * ne, c, r)


@pytest.mark.parametrize("c,kernel", [(512, "fused_pair_kernel/hca/cache"),
                                      (384, "fused_pool_kernel/hca/cache")])
def test_hca_fused_cache(c, kernel):
    batch, n, d, r = 2, 128 * 9 + 5, 192, 64
    h = synth.fused_inputs("hca", batch, n, d, c, 128, seed=c)
    t = _dev(h)
    inv = _inv_freq(r)
    ne = n // 128
    nb, rb, nope, rope = _guarded_cache_outs(batch * ne, c, r)
    kvc.hca_compress_fused_proj_cache(t["H"], t["W_kv"], t["W_z"], t["B"], batch, n, r,
                                      torch.from_numpy(inv).cuda(), pos_stride=128.0,
                                      pos_offset=63.5, fp8_scale=1.0, out_nope=nope, out_rope=rope)
    assert kvc.last_kernel() == kernel
    assert kvc.device_status() == kvc.KVC_OK
    ent = O.hca_compress_fused(h["H"], h["W_kv"], h["W_z"], h["B"], batch, n, 128)
    _compare(nope.view(batch, ne, c - r), rope.view(batch, ne, r), ent, r, inv, 128.0, 63.5, 1.0,
             f"hca fused cache c={c}")
    _guards_ok(nb, rb, batch * ne, c, r)


def test_hca_fused_cache_large_positions_and_saturation():
    """Positions near 2^20 exercise the fp64 angle reduction; a scale of 2000 saturates
    many E4M3 codes at 448."""
    batch, n, d, c, r = 1, 128 * 12, 128, 512, 64
    h = synth.fused_inputs("hca", batch, n, d, c, 128, seed=7)
    t = _dev(h)
    inv = _inv_freq(r)
    nope, rope = kvc.hca_compress_fused_proj_cache(t["H"], t["W_kv"], t["W_z"], t["B"], batch, n, r,
                                                   torch.from_numpy(inv).cuda(), pos_stride=128.0,
                                                   pos_offset=1048000.5, fp8_scale=2000.0)
    assert kvc.device_status() == kvc.KVC_OK
    ent = O.hca_compress_fused(h["H"], h["W_kv"], h["W_z"], h["B"], batch, n, 128)
    _compare(nope, rope, ent, r, inv, 128.0, 1048000.5, 2000.0, "hca fused cache saturation")
    assert np.any(np.abs(_fp8_values(nope)) == 448.0)


def test_fused_cache_agrees_with_plain_fused():
    """The cache-layout epilogue rounds the same fp32 entries that the plain epilogue
    stores: the RoPE part of r = c at position 0 (no rotation) equals the plain bf16
    output bit for bit."""
    batch, n, d, c = 1, 4 * 300, 256, 256
    h = synth.fused_inputs("csa", batch, n, d, c, 4, seed=9)
    t = _dev(h)
    inv = torch.from_numpy(_inv_freq(c)).cuda()
    _, rope = kvc.csa_compress_fused_proj_cache(t["H"], t["W_kva"], t["W_kvb"], t["W_za"],
                                                t["W_zb"], t["Ba"], t["Bb"], batch, n, c, inv,
                                                pos_stride=0.0, pos_offset=0.0)
    plain = kvc.csa_compress_fused_proj(t["H"], t["W_kva"], t["W_kvb"], t["W_za"], t["W_zb"],
                                        t["Ba"], t["Bb"], batch, n, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(rope, plain)


def test_csa_fused_cache_n32768_d7168_sampled():
    """The fused CSA workload (H [32768, 7168]) in the cache layout with r = 64: sampled
    entries (random, first and last, tile and piece boundaries) against the oracle entry
    evaluated on the rows it reads, then put in the cache layout at its own position."""
    w = synth.WORKLOADS["csa_fused_n32768_d7168"]
    n, c, r = w["n"], w["c"], 64
    t = synth.fused_inputs_torch("csa", 1, n, w["d"], c, 4, seed=3)
    inv = _inv_freq(r)
    nope, rope = kvc.csa_compress_fused_proj_cache(t["H"], t["W_kva"], t["W_kvb"], t["W_za"],
                                                   t["W_zb"], t["Ba"], t["Bb"], 1, n, r,
                                                   torch.from_numpy(inv).cuda())
    assert kvc.device_status() == kvc.KVC_OK
    ne = n // 4
    rng = np.random.default_rng(3)
    ents = set(rng.choice(ne, size=120, replace=False).tolist()) | {0, 1, ne - 1}
    ents |= {min(ne - 1, 63 * k + dd) for k in range(1, 6) for dd in (-1, 0, 1)}
    ents |= {min(ne - 1, (ne * q) // 74 + dd) for q in range(1, 4) for dd in (-1, 0, 1)}
    ents = sorted(ents)
    Ws = {k: host64(v) for k, v in t.items() if k.startswith("W") or k.startswith("B")}
    refs = []
    for i in ents:
        lo = 4 * (i - 1) if i > 0 else 0
        rows = host64(t["H"][lo:4 * i + 4])
        refs.append(O.csa_compress_fused(rows, Ws["W_kva"], Ws["W_kvb"], Ws["W_za"], Ws["W_zb"],
                                         Ws["Ba"], Ws["Bb"], 1, 4 * i + 4 - lo, 4, True,
                                         entries=[(0, 1 if i > 0 else 0)])[0])
    refs = np.array(refs)
    pos = 1.5 + 4.0 * np.array(ents, dtype=np.float64)
    ref_nope = O.round_e4m3(refs[:, :c - r])
    ref_rope = O.rope_pairs(refs[:, c - r:], pos, inv.astype(np.float64))
    idx = torch.as_tensor(ents, device="cuda")
    _check_fp8(_fp8_values(nope[0, idx]), ref_nope, "csa fused cache sampled nope")
    check_close(rope[0, idx], ref_rope, "bf16", "csa fused cache sampled rope")
    del t
    torch.cuda.empty_cache()
