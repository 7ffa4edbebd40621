"""Every kernel behind the compressor's entry points, reached through the C ABI on purpose.

The calls pick a kernel by problem size (tasks per SM, window length, channel count, dtype):
each case below is sized to land on one of them, asserts through kvc_last_kernel() that it
did, and compares every output element with the fp64 oracle.  Outputs are written into
buffers with canary guard bands on both sides that must come back untouched (nothing is
written before or past the output)."""

from __future__ import annotations

import functools

import numpy as np
import pytest
import torch

from gpu_util import check_close, dev, tdtype
from kv_token_compressor_b200 import kvc, synth
from oracle import compressor as O

pytestmark = pytest.mark.gpu

GUARD = 64          # elements on each side: keeps the output 16-byte aligned
CANARY = -1280.0    # exact in bf16 and fp32


def guarded(shape, dtype):
    numel = int(np.prod(shape))
    buf = torch.full((numel + 2 * GUARD,), CANARY, dtype=dtype, device="cuda")
    return buf, buf[GUARD:GUARD + numel].view(shape)


def assert_guards(buf, numel, what):
    head, tail = buf[:GUARD], buf[GUARD + numel:]
    assert bool(torch.all(head == CANARY)), f"{what}: written before the output"
    assert bool(torch.all(tail == CANARY)), f"{what}: written past the output"


@functools.lru_cache(maxsize=4)
def _stream(mode, batch, n, c, m, dt, seed):
    return synth.stream_inputs(mode, batch, n, c, m, dt, seed=seed)


def run_csa(batch, n, c, m, overlap, in_dt, out_dt, seed=0):
    d = _stream("csa", batch, n, c, m, in_dt, seed)
    t = {k: dev(v, in_dt) if v.ndim == 3 else dev(v, "f32") for k, v in d.items()}
    shape = (batch, n // m, c)
    buf, out = guarded(shape, tdtype(out_dt))
    kvc.csa_compress(t["Ca"], t["Cb"] if overlap else None, t["Za"], t["Zb"] if overlap else None,
                     t["Ba"], t["Bb"] if overlap else None, m=m, overlap=overlap, out=out,
                     out_dtype=tdtype(out_dt))
    name = kvc.last_kernel()
    assert kvc.device_status() == kvc.KVC_OK
    if overlap:
        ref = O.csa_compress(d["Ca"], d["Cb"], d["Za"], d["Zb"], d["Ba"], d["Bb"], m, True)
    else:
        ref = O.csa_compress(d["Ca"], None, d["Za"], None, d["Ba"], None, m, False)
    what = f"csa {batch}x{n}x{c} m={m} ov={overlap} {in_dt}->{out_dt}"
    check_close(out, ref, out_dt, what)
    assert_guards(buf, out.numel(), what)
    return name


def run_hca(batch, n, c, m, in_dt, out_dt, seed=0):
    d = _stream("hca", batch, n, c, m, in_dt, seed)
    shape = (batch, n // m, c)
    buf, out = guarded(shape, tdtype(out_dt))
    kvc.hca_compress(dev(d["C"], in_dt), dev(d["Z"], in_dt), dev(d["B"], "f32"), m=m, out=out,
                     out_dtype=tdtype(out_dt))
    name = kvc.last_kernel()
    assert kvc.device_status() == kvc.KVC_OK
    what = f"hca {batch}x{n}x{c} m={m} {in_dt}->{out_dt}"
    check_close(out, O.hca_compress(d["C"], d["Z"], d["B"], m), out_dt, what)
    assert_guards(buf, out.numel(), what)
    return name


# Dense CSA.  The TMA-fed kernel serves up to 16 tasks (8 entries x one channel slab of 128
# bf16 / 64 fp32 channels) per SM; beyond that the register-staged kernel, compiled with
# the row stride as a constant at c = 512 (compressed KV) and c = 128 (indexer keys).
CSA_DISPATCH = [
    # kernel, batch, n, c, m, overlap, in, out
    ("csa_tma_kernel", 1, 4 * 4096 + 3, 512, 4, True, "bf16", "bf16"),
    ("csa_small_m_kernel/c512", 1, 1 << 17, 512, 4, True, "f32", "f32"),
    ("csa_small_m_kernel/c512", 1, 1 << 17, 512, 4, True, "f32", "bf16"),
    ("csa_small_m_kernel/c512", 2, 4 * 20000 + 1, 512, 4, True, "bf16", "bf16"),
    ("csa_small_m_kernel/c128", 1, 1 << 18, 128, 4, True, "bf16", "bf16"),
    ("csa_small_m_kernel/c128", 1, 1 << 18, 128, 4, True, "bf16", "f32"),
    ("csa_small_m_kernel/c128", 3, 4 * 30000 + 2, 128, 4, True, "f32", "f32"),
    ("csa_small_m_kernel", 1, 1 << 17, 256, 4, True, "bf16", "bf16"),
    ("csa_small_m_kernel", 2, 51, 24, 2, True, "f32", "bf16"),
    ("csa_small_m_kernel", 2, 4 * 33 + 1, 520, 4, False, "bf16", "f32"),
    # two-segment windows of other lengths: the register-staged window kernel, with 16, 4
    # or 1 row groups per window as the task count grows (windows of <= 8 rows: always 1)
    ("window_pool_kernel/rg16", 2, 8 * 21 + 5, 72, 8, True, "f32", "f32"),
    ("window_pool_kernel/rg4", 1, 8 * 4000, 64, 8, True, "f32", "f32"),
    ("window_pool_kernel/rg1", 1, 8 * 15000 + 3, 64, 8, True, "f32", "bf16"),
    ("window_pool_kernel/rg1", 1, 3 * 40 + 2, 16, 3, True, "bf16", "bf16"),
]


@pytest.mark.parametrize("kernel,batch,n,c,m,overlap,in_dt,out_dt", CSA_DISPATCH,
                         ids=[f"{k}-{b}x{n}x{c}-m{m}-{i}-{o}" for k, b, n, c, m, _, i, o in CSA_DISPATCH])
def test_csa_dispatch(kernel, batch, n, c, m, overlap, in_dt, out_dt):
    assert run_csa(batch, n, c, m, overlap, in_dt, out_dt, seed=n + c) == kernel


# Dense single-segment windows (HCA).  Windows of 32 or more rows whose bias fits take
# the TMA-fed window kernel; the others the register-staged kernels: windows of <= 8 rows
# one per thread, longer ones pipelined over 16, 8 or 4 row groups, or one per thread once
# there are many.
HCA_DISPATCH = [
    ("window_tma_kernel", 1, 128 * 74, 512, 128, "bf16", "bf16"),
    ("window_tma_kernel", 2, 64 * 300 + 9, 256, 64, "f32", "f32"),
    ("window_pipe_kernel/rg16", 1, 16 * 100, 64, 16, "f32", "f32"),
    ("window_pipe_kernel/rg8", 1, 16 * 1000 + 5, 64, 16, "f32", "bf16"),
    ("window_pipe_kernel/rg4", 1, 16 * 4000, 64, 16, "f32", "f32"),
    ("window_pool_kernel/rg1", 1, 16 * 15000, 64, 16, "f32", "f32"),
    ("window_pool_kernel/rg1", 1, 7 * 11, 512, 7, "bf16", "f32"),
    ("window_pipe_kernel/rg16", 1, 256 * 20, 128, 256, "bf16", "bf16"),
]


@pytest.mark.parametrize("kernel,batch,n,c,m,in_dt,out_dt", HCA_DISPATCH,
                         ids=[f"{k}-{b}x{n}x{c}-m{m}-{i}-{o}" for k, b, n, c, m, i, o in HCA_DISPATCH])
def test_hca_dispatch(kernel, batch, n, c, m, in_dt, out_dt):
    assert run_hca(batch, n, c, m, in_dt, out_dt, seed=n + c + 1) == kernel


def test_scalar_dispatch():
    d = synth.scalar_inputs("csa", 2, 4 * 300 + 1, 136, 4, "bf16", seed=2)
    t = {k: dev(v, "bf16") if k in ("Ca", "Cb", "za", "zb") else dev(v, "f32") for k, v in d.items()}
    buf, out = guarded((2, 300, 136), torch.bfloat16)
    kvc.csa_compress_scalar_logits(t["Ca"], t["Cb"], t["za"], t["zb"], t["ba"], t["bb"], m=4,
                                   out=out)
    assert kvc.last_kernel() == "scalar_small_m_kernel"
    torch.cuda.synchronize()
    ref = O.csa_compress_scalar(d["Ca"], d["Cb"], d["za"], d["zb"], d["ba"], d["bb"], 4, True)
    check_close(out, ref, "bf16", "csa scalar")
    assert_guards(buf, out.numel(), "csa scalar")

    h = synth.scalar_inputs("hca", 1, 128 * 40 + 3, 264, 128, "f32", seed=3)
    buf, out = guarded((1, 40, 264), torch.float32)
    kvc.hca_compress_scalar_logits(dev(h["C"], "f32"), dev(h["z"], "f32"), dev(h["b"], "f32"),
                                   m=128, out=out)
    assert kvc.last_kernel() == "scalar_pool_kernel"
    torch.cuda.synchronize()
    check_close(out, O.hca_compress_scalar(h["C"], h["z"], h["b"], 128), "f32", "hca scalar")
    assert_guards(buf, out.numel(), "hca scalar")


# Entry lists (CSA, m = 4, overlap) take the register-staged kernel (one window per thread)
# at every row width, input and output type and list length.
CSA_LISTED = [
    # kernel, c, in, out, sequence lengths, entry step
    ("csa_small_m_kernel", 128, "bf16", "f32", [4 * 50 + 1, 4 * 3, 4 * 77], 3),
    ("csa_small_m_kernel", 256, "bf16", "bf16", [4 * 20, 4 * 91 + 2, 5, 4 * 7], 1),
    ("csa_small_m_kernel", 512, "bf16", "bf16", [4 * 33 + 3, 4 * 64, 4], 1),
    ("csa_small_m_kernel", 64, "f32", "f32", [4 * 40, 4 * 9 + 1], 1),
    ("csa_small_m_kernel", 128, "f32", "bf16", [4 * 17, 4 * 50 + 3], 2),
    ("csa_small_m_kernel", 256, "f32", "f32", [4 * 70 + 1, 4 * 2], 1),
    ("csa_small_m_kernel", 136, "bf16", "f32", [4 * 50 + 1, 4 * 3, 4 * 77], 3),
    ("csa_small_m_kernel", 512, "bf16", "bf16", [4 * 6001 + 2], 1),  # a long list
]


@pytest.mark.parametrize("kernel,c,in_dt,out_dt,lens,step", CSA_LISTED,
                         ids=[f"{k}-c{c}-{i}-{o}-{len(L)}seq" for k, c, i, o, L, _ in CSA_LISTED])
def test_csa_listed_dispatch(kernel, c, in_dt, out_dt, lens, step):
    d = synth.stream_inputs("csa", 1, sum(lens), c, 4, in_dt, seed=9 + c)
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]])
    ents = [(s, e) for s, L in enumerate(lens) for e in range(0, L // 4, step)]
    ents = ents[::-1]  # list order is not sequence order
    t = {k: dev(v[0], in_dt) if v.ndim == 3 else dev(v, "f32") for k, v in d.items()}
    ss = torch.tensor([int(starts[s]) for s, _ in ents], dtype=torch.int64, device="cuda")
    sl = torch.tensor([lens[s] for s, _ in ents], dtype=torch.int64, device="cuda")
    en = torch.tensor([e for _, e in ents], dtype=torch.int64, device="cuda")
    buf, out = guarded((len(ents), c), tdtype(out_dt))
    kvc.csa_compress_entries(t["Ca"], t["Cb"], t["Za"], t["Zb"], t["Ba"], t["Bb"], ss, sl, en, m=4,
                             out=out, out_dtype=tdtype(out_dt))
    assert kvc.last_kernel() == kernel
    assert kvc.device_status() == kvc.KVC_OK
    ref = {}
    for s, L in enumerate(lens):  # every entry of a sequence at once
        q = slice(int(starts[s]), int(starts[s]) + L)
        if L // 4:
            ref[s] = O.csa_compress(d["Ca"][:, q], d["Cb"][:, q], d["Za"][:, q], d["Zb"][:, q],
                                    d["Ba"], d["Bb"], 4, True)[0]
    check_close(out, np.array([ref[s][e] for s, e in ents]), out_dt, f"csa listed c={c}")
    assert_guards(buf, out.numel(), "csa listed")


def test_hca_listed_dispatch():
    c = 128
    h = synth.stream_inputs("hca", 1, 128 * 12, c, 128, "bf16", seed=10)
    th = {k: dev(v[0], "bf16") if v.ndim == 3 else dev(v, "f32") for k, v in h.items()}
    idx = torch.arange(12, dtype=torch.int64, device="cuda")
    buf, out = guarded((12, c), torch.bfloat16)
    kvc.hca_compress_entries(th["C"], th["Z"], th["B"], torch.zeros_like(idx),
                             torch.full_like(idx, 128 * 12), idx, m=128, out=out)
    assert kvc.last_kernel() == "window_pool_kernel/rg1"
    assert kvc.device_status() == kvc.KVC_OK
    check_close(out, O.hca_compress(h["C"], h["Z"], h["B"], 128)[0], "bf16", "hca listed")
    assert_guards(buf, out.numel(), "hca listed")


def _fused_dev(h):
    return {k: torch.from_numpy(np.ascontiguousarray(v)).cuda().to(
        torch.float32 if k.startswith("B") else torch.bfloat16) for k, v in h.items()}


@pytest.mark.parametrize("kernel,c", [("fused_pair_kernel/hca", 512), ("fused_pool_kernel/hca", 384)])
def test_fused_hca_dispatch(kernel, c):
    """An even number of 128-channel groups pairs them over a CTA pair; an odd number takes
    the single-CTA kernel."""
    batch, n, d = 2, 128 * 6 + 5, 192
    h = synth.fused_inputs("hca", batch, n, d, c, 128, seed=c)
    t = _fused_dev(h)
    buf, out = guarded((batch, n // 128, c), torch.bfloat16)
    kvc.hca_compress_fused_proj(t["H"], t["W_kv"], t["W_z"], t["B"], batch, n, m=128, out=out)
    assert kvc.last_kernel() == kernel
    assert kvc.device_status() == kvc.KVC_OK
    ref = O.hca_compress_fused(h["H"], h["W_kv"], h["W_z"], h["B"], batch, n, 128)
    check_close(out, ref, "bf16", f"hca fused c={c}")
    assert_guards(buf, out.numel(), f"hca fused c={c}")


def test_fused_csa_dispatch():
    batch, n, d, c = 2, 4 * 900 + 3, 128, 256
    h = synth.fused_inputs("csa", batch, n, d, c, 4, seed=5)
    t = _fused_dev(h)
    buf, out = guarded((batch, n // 4, c), torch.float32)
    kvc.csa_compress_fused_proj(t["H"], t["W_kva"], t["W_kvb"], t["W_za"], t["W_zb"], t["Ba"],
                                t["Bb"], batch, n, m=4, out=out, out_dtype=torch.float32)
    assert kvc.last_kernel() == "fused_pair_kernel/csa"
    assert kvc.device_status() == kvc.KVC_OK
    ref = O.csa_compress_fused(h["H"], h["W_kva"], h["W_kvb"], h["W_za"], h["W_zb"], h["Ba"],
                               h["Bb"], batch, n, 4, True)
    check_close(out, ref, "f32", "csa fused")
    assert_guards(buf, out.numel(), "csa fused")


def test_last_kernel_is_per_thread():
    """The record belongs to the calling host thread."""
    import threading

    d = _stream("hca", 1, 128 * 74, 512, 128, "bf16", 0)
    t = {k: dev(v, "bf16") if v.ndim == 3 else dev(v, "f32") for k, v in d.items()}
    kvc.hca_compress(t["C"], t["Z"], t["B"], m=128)
    assert kvc.last_kernel() == "window_tma_kernel"
    seen = []

    def other():
        seen.append(kvc.last_kernel())
        x = dev(np.ones((1, 64, 64), np.float32), "f32")
        b = dev(np.zeros((4, 64), np.float32), "f32")
        kvc.csa_compress(x, x, x, x, b, b, m=4)
        seen.append(kvc.last_kernel())

    th = threading.Thread(target=other)
    th.start()
    th.join()
    torch.cuda.synchronize()
    assert seen == ["", "csa_tma_kernel"]
    assert kvc.last_kernel() == "window_tma_kernel"


def test_concurrent_threads_with_different_windows():
    """Two host threads run the same kernel (the TMA-fed window kernel) with different
    shared-memory needs (m = 64 and m = 128), 100 calls each on their own streams: every
    launch succeeds and every result equals the oracle's (to the output's rounding)."""
    import threading

    cases = {}
    for m in (64, 128):
        d = synth.stream_inputs("hca", 1, m * 200 + 3, 256, m, "bf16", seed=m)
        t = {k: dev(v, "bf16") if v.ndim == 3 else dev(v, "f32") for k, v in d.items()}
        cases[m] = (d, t, O.hca_compress(d["C"], d["Z"], d["B"], m))
    results, errors = {64: [], 128: []}, []

    def worker(m):
        try:
            d, t, _ = cases[m]
            st = torch.cuda.Stream()
            with torch.cuda.stream(st):
                for _ in range(100):
                    out = kvc.hca_compress(t["C"], t["Z"], t["B"], m=m, stream=st)
                    results[m].append(out)
                    if kvc.last_kernel() != "window_tma_kernel":
                        errors.append(f"m={m}: {kvc.last_kernel()}")
            st.synchronize()
        except Exception as e:  # reported below
            errors.append(f"m={m}: {e!r}")

    ths = [threading.Thread(target=worker, args=(m,)) for m in (64, 128)]
    for th in ths:
        th.start()
    for th in ths:
        th.join()
    torch.cuda.synchronize()
    assert not errors, errors[:3]
    assert kvc.device_status() == kvc.KVC_OK
    for m, outs in results.items():
        assert len(outs) == 100
        check_close(outs[0], cases[m][2], "bf16", f"threads m={m}")
        for o in outs[1:]:
            assert torch.equal(o, outs[0]), f"m={m}: results differ between calls"
