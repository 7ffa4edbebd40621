"""The C-ABI library on the host: it loads, exports every entry point that
include/kvc.h declares, and rejects bad arguments before touching the GPU.

Only argument errors that the library detects before its first CUDA call are
exercised here (no device is needed and no pointer is ever dereferenced)."""

import ctypes
import os
import re
import subprocess
import sys

import pytest

from kv_token_compressor_b200 import kvc

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kvc.h")

# Fake, never-dereferenced device addresses (16-byte aligned unless stated).
A = 0x7F0000000000
MIS = A + 8


def header_entry_points():
    src = open(HEADER).read()
    return re.findall(r"KVC_API\s+[\w\s\*]+?\b(\w+)\s*\(", src)


@pytest.fixture(scope="module")
def L():
    from kv_token_compressor_b200 import build

    build.build()
    return kvc.lib()


def test_header_declares_the_boundary():
    names = set(header_entry_points())
    assert {"csa_compress", "hca_compress", "csa_compress_fused_proj", "hca_compress_fused_proj",
            "kvc_num_entries", "kvc_status_string", "kvc_device_status"} <= names


def test_every_declared_symbol_is_exported(L):
    out = subprocess.run(["nm", "-D", "--defined-only", kvc.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    for name in header_entry_points():
        assert name in exported, name
        assert hasattr(L, name)
    assert set(kvc.SIGNATURES) == set(header_entry_points())


def test_num_entries_bit_exact(L):
    for n in list(range(0, 300)) + [1 << 20, 10**6, (1 << 40) + 3]:
        for m in (1, 2, 3, 4, 7, 8, 128, 1000):
            assert L.kvc_num_entries(n, m) == n // m
    assert L.kvc_num_entries(-1, 4) == -1
    assert L.kvc_num_entries(10, 0) == -1
    assert L.kvc_num_entries(10, -4) == -1


def test_status_strings(L):
    for code in range(10):
        s = kvc.status_string(code)
        assert s.startswith("KVC_")
    assert kvc.status_string(99) == "KVC_ERR_UNKNOWN"


def csa(L, **kw):
    a = dict(Ca=A, Cb=A, Za=A, Zb=A, in_dt=kvc.KVC_BF16, Ba=A, Bb=A, batch=1, n=1024, c=512, m=4,
             overlap=1, out=A, out_dt=kvc.KVC_BF16)
    a.update(kw)
    return L.csa_compress(a["Ca"], a["Cb"], a["Za"], a["Zb"], a["in_dt"], a["Ba"], a["Bb"],
                          a["batch"], a["n"], a["c"], a["m"], a["overlap"], a["out"], a["out_dt"],
                          None)


def hca(L, **kw):
    a = dict(C=A, Z=A, in_dt=kvc.KVC_BF16, B=A, batch=1, n=65536, c=512, m=128, out=A,
             out_dt=kvc.KVC_BF16)
    a.update(kw)
    return L.hca_compress(a["C"], a["Z"], a["in_dt"], a["B"], a["batch"], a["n"], a["c"], a["m"],
                          a["out"], a["out_dt"], None)


def fused_csa(L, **kw):
    a = dict(H=A, Wa=A, Wb=A, Za=A, Zb=A, Ba=A, Bb=A, batch=1, n=4096, d=7168, c=512, m=4,
             overlap=1, out=A, out_dt=kvc.KVC_BF16)
    a.update(kw)
    return L.csa_compress_fused_proj(a["H"], a["Wa"], a["Wb"], a["Za"], a["Zb"], a["Ba"], a["Bb"],
                                     a["batch"], a["n"], a["d"], a["c"], a["m"], a["overlap"],
                                     a["out"], a["out_dt"], None)


def fused_hca(L, **kw):
    a = dict(H=A, Wk=A, Wz=A, B=A, batch=1, n=4096, d=4096, c=512, m=128, out=A,
             out_dt=kvc.KVC_BF16)
    a.update(kw)
    return L.hca_compress_fused_proj(a["H"], a["Wk"], a["Wz"], a["B"], a["batch"], a["n"], a["d"],
                                     a["c"], a["m"], a["out"], a["out_dt"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(in_dt=7), kvc.KVC_ERR_DTYPE),
    (dict(out_dt=-1), kvc.KVC_ERR_DTYPE),
    (dict(n=-1), kvc.KVC_ERR_SHAPE),
    (dict(batch=-2), kvc.KVC_ERR_SHAPE),
    (dict(c=-8), kvc.KVC_ERR_SHAPE),
    (dict(c=500), kvc.KVC_ERR_SHAPE),
    (dict(m=0), kvc.KVC_ERR_SHAPE),
    (dict(overlap=2), kvc.KVC_ERR_SHAPE),
    (dict(batch=1 << 40, n=1 << 20, c=1 << 10), kvc.KVC_ERR_SHAPE),
    (dict(Ca=None), kvc.KVC_ERR_NULL),
    (dict(Zb=None), kvc.KVC_ERR_NULL),
    (dict(Bb=None), kvc.KVC_ERR_NULL),
    (dict(out=None), kvc.KVC_ERR_NULL),
    (dict(Ca=MIS), kvc.KVC_ERR_ALIGN),
    (dict(Zb=MIS), kvc.KVC_ERR_ALIGN),
    (dict(out=MIS), kvc.KVC_ERR_ALIGN),
    (dict(Ba=A + 2), kvc.KVC_ERR_ALIGN),
    (dict(m=200), kvc.KVC_ERR_UNSUPPORTED),
])
def test_csa_rejects_before_launch(L, kw, status):
    assert csa(L, **kw) == status


def test_csa_overlap_off_ignores_b_pointers(L):
    # With overlap = 0 the b-stream pointers may be NULL: validation passes them.
    st = csa(L, overlap=0, Cb=None, Zb=None, Bb=None, Ca=MIS)
    assert st == kvc.KVC_ERR_ALIGN  # it got as far as checking the a-stream pointer


@pytest.mark.parametrize("kw", [dict(n=3), dict(n=0), dict(batch=0), dict(c=0)])
def test_csa_empty_problem_is_ok_and_touches_nothing(L, kw):
    assert csa(L, Ca=None, Cb=None, Za=None, Zb=None, Ba=None, Bb=None, out=None, **kw) == kvc.KVC_OK


@pytest.mark.parametrize("kw,status", [
    (dict(in_dt=2), kvc.KVC_ERR_DTYPE),
    (dict(n=-5), kvc.KVC_ERR_SHAPE),
    (dict(c=12), kvc.KVC_ERR_SHAPE),
    (dict(m=0), kvc.KVC_ERR_SHAPE),
    (dict(Z=None), kvc.KVC_ERR_NULL),
    (dict(B=None), kvc.KVC_ERR_NULL),
    (dict(C=MIS), kvc.KVC_ERR_ALIGN),
    (dict(m=321), kvc.KVC_ERR_UNSUPPORTED),
])
def test_hca_rejects_before_launch(L, kw, status):
    assert hca(L, **kw) == status


def test_hca_empty(L):
    assert hca(L, n=127, C=None, Z=None, B=None, out=None) == kvc.KVC_OK


@pytest.mark.parametrize("kw,status", [
    (dict(out_dt=5), kvc.KVC_ERR_DTYPE),
    (dict(d=7160), kvc.KVC_ERR_SHAPE),
    (dict(c=448), kvc.KVC_ERR_SHAPE),
    (dict(m=0), kvc.KVC_ERR_SHAPE),
    (dict(overlap=3), kvc.KVC_ERR_SHAPE),
    (dict(H=None), kvc.KVC_ERR_NULL),
    (dict(Zb=None), kvc.KVC_ERR_NULL),
    (dict(Bb=None), kvc.KVC_ERR_NULL),
    (dict(H=MIS), kvc.KVC_ERR_ALIGN),
    (dict(Wb=MIS), kvc.KVC_ERR_ALIGN),
])
def test_fused_csa_rejects_before_launch(L, kw, status):
    assert fused_csa(L, **kw) == status


@pytest.mark.parametrize("kw,status", [
    (dict(d=100), kvc.KVC_ERR_SHAPE),
    (dict(c=200), kvc.KVC_ERR_SHAPE),
    (dict(Wz=None), kvc.KVC_ERR_NULL),
    (dict(Wk=MIS), kvc.KVC_ERR_ALIGN),
])
def test_fused_hca_rejects_before_launch(L, kw, status):
    assert fused_hca(L, **kw) == status


@pytest.mark.parametrize("kw,status", [
    (dict(m=8), kvc.KVC_ERR_UNSUPPORTED),
    (dict(m=2), kvc.KVC_ERR_UNSUPPORTED),
    (dict(overlap=0), kvc.KVC_ERR_UNSUPPORTED),
])
def test_fused_csa_only_the_pages_compressor(L, kw, status):
    """The tensor-core path implements CSA with m = 4 and overlap only; other valid
    ratios are refused before any CUDA call (fake pointers are never dereferenced)."""
    assert fused_csa(L, **kw) == status


@pytest.mark.parametrize("m", [64, 4, 256])
def test_fused_hca_only_m_128(L, m):
    assert fused_hca(L, m=m) == kvc.KVC_ERR_UNSUPPORTED


def fused_csa_cache(L, **kw):
    a = dict(H=A, Wa=A, Wb=A, Za=A, Zb=A, Ba=A, Bb=A, batch=1, n=4096, d=7168, c=512, m=4,
             overlap=1, r=64, inv=A, stride=4.0, offset=1.5, scale=1.0, nope=A, rope=A)
    a.update(kw)
    return L.csa_compress_fused_proj_cache(a["H"], a["Wa"], a["Wb"], a["Za"], a["Zb"], a["Ba"],
                                           a["Bb"], a["batch"], a["n"], a["d"], a["c"], a["m"],
                                           a["overlap"], a["r"], a["inv"], a["stride"],
                                           a["offset"], a["scale"], a["nope"], a["rope"], None)


def fused_hca_cache(L, **kw):
    a = dict(H=A, Wk=A, Wz=A, B=A, batch=1, n=4096, d=4096, c=512, m=128, r=64, inv=A,
             stride=128.0, offset=63.5, scale=1.0, nope=A, rope=A)
    a.update(kw)
    return L.hca_compress_fused_proj_cache(a["H"], a["Wk"], a["Wz"], a["B"], a["batch"], a["n"],
                                           a["d"], a["c"], a["m"], a["r"], a["inv"], a["stride"],
                                           a["offset"], a["scale"], a["nope"], a["rope"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(r=12), kvc.KVC_ERR_SHAPE),
    (dict(r=520), kvc.KVC_ERR_SHAPE),
    (dict(r=-8), kvc.KVC_ERR_SHAPE),
    (dict(scale=float("nan")), kvc.KVC_ERR_SHAPE),
    (dict(inv=None), kvc.KVC_ERR_NULL),
    (dict(nope=None), kvc.KVC_ERR_NULL),
    (dict(rope=MIS), kvc.KVC_ERR_ALIGN),
    (dict(inv=A + 2), kvc.KVC_ERR_ALIGN),
    (dict(m=8), kvc.KVC_ERR_UNSUPPORTED),
    (dict(overlap=0), kvc.KVC_ERR_UNSUPPORTED),
    (dict(d=100), kvc.KVC_ERR_SHAPE),
    (dict(H=None), kvc.KVC_ERR_NULL),
])
def test_fused_csa_cache_rejects_before_launch(L, kw, status):
    assert fused_csa_cache(L, **kw) == status


@pytest.mark.parametrize("kw,status", [
    (dict(r=4), kvc.KVC_ERR_SHAPE),
    (dict(rope=None), kvc.KVC_ERR_NULL),
    (dict(nope=MIS), kvc.KVC_ERR_ALIGN),
    (dict(m=64), kvc.KVC_ERR_UNSUPPORTED),
    (dict(Wz=None), kvc.KVC_ERR_NULL),
])
def test_fused_hca_cache_rejects_before_launch(L, kw, status):
    assert fused_hca_cache(L, **kw) == status


def test_fused_cache_optional_parts_and_empty(L):
    # an empty problem touches nothing; r = 0 needs no RoPE output or frequencies, r = c
    # no E4M3 output (checked up to the device-memory check, which fails without a GPU)
    assert fused_csa_cache(L, n=3, H=None, nope=None, rope=None) == kvc.KVC_OK
    assert fused_hca_cache(L, batch=0, H=None, nope=None, rope=None) == kvc.KVC_OK
    for kw in (dict(r=0, rope=None, inv=None), dict(r=512, nope=None)):
        assert fused_csa_cache(L, **kw) not in (kvc.KVC_ERR_NULL, kvc.KVC_ERR_SHAPE,
                                                kvc.KVC_ERR_ALIGN)


def test_prepared_bias_workspace_size(L):
    # header, raw bias, and per slab (m + 1) * SC + 4 floats (SC = 128 bf16, 64 fp32)
    raw = -(-128 * 512 * 4 // 256) * 256
    assert L.hca_bias_workspace_bytes(512, 128, kvc.KVC_BF16) == 256 + raw + 4 * (129 * 128 + 4) * 4
    assert L.hca_bias_workspace_bytes(512, 128, kvc.KVC_F32) == 256 + raw + 8 * (129 * 64 + 4) * 4
    assert L.hca_bias_workspace_bytes(8, 1, kvc.KVC_BF16) == 256 + 256 + (2 * 128 + 4) * 4
    for bad in ((0, 128, kvc.KVC_BF16), (512, 0, kvc.KVC_BF16), (512, 128, 7)):
        assert L.hca_bias_workspace_bytes(*bad) == -1


def prep(L, **kw):
    need = L.hca_bias_workspace_bytes(512, 128, kvc.KVC_BF16)
    a = dict(B=A, c=512, m=128, dt=kvc.KVC_BF16, ws=A, nbytes=need)
    a.update(kw)
    return L.hca_prepare_bias(a["B"], a["c"], a["m"], a["dt"], a["ws"], a["nbytes"], None)


def hca_prep(L, **kw):
    need = L.hca_bias_workspace_bytes(512, 128, kvc.KVC_BF16)
    a = dict(C=A, Z=A, dt=kvc.KVC_BF16, ws=A, nbytes=need, batch=1, n=65536, c=512, m=128, out=A,
             out_dt=kvc.KVC_BF16)
    a.update(kw)
    return L.hca_compress_prepared(a["C"], a["Z"], a["dt"], a["ws"], a["nbytes"], a["batch"],
                                   a["n"], a["c"], a["m"], a["out"], a["out_dt"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(dt=9), kvc.KVC_ERR_DTYPE),
    (dict(c=12), kvc.KVC_ERR_SHAPE),
    (dict(c=0), kvc.KVC_ERR_SHAPE),
    (dict(m=0), kvc.KVC_ERR_SHAPE),
    (dict(m=321), kvc.KVC_ERR_UNSUPPORTED),
    (dict(nbytes=1000), kvc.KVC_ERR_SHAPE),
    (dict(B=None), kvc.KVC_ERR_NULL),
    (dict(ws=None), kvc.KVC_ERR_NULL),
    (dict(ws=A + 16), kvc.KVC_ERR_ALIGN),
    (dict(B=A + 2), kvc.KVC_ERR_ALIGN),
])
def test_prepare_bias_rejects_before_launch(L, kw, status):
    assert prep(L, **kw) == status


@pytest.mark.parametrize("kw,status", [
    (dict(out_dt=4), kvc.KVC_ERR_DTYPE),
    (dict(n=-1), kvc.KVC_ERR_SHAPE),
    (dict(c=100), kvc.KVC_ERR_SHAPE),
    (dict(nbytes=4096), kvc.KVC_ERR_SHAPE),
    (dict(m=400), kvc.KVC_ERR_UNSUPPORTED),
    (dict(ws=None), kvc.KVC_ERR_NULL),
    (dict(Z=None), kvc.KVC_ERR_NULL),
    (dict(ws=A + 64), kvc.KVC_ERR_ALIGN),
    (dict(out=MIS), kvc.KVC_ERR_ALIGN),
])
def test_hca_prepared_rejects_before_launch(L, kw, status):
    assert hca_prep(L, **kw) == status


def test_hca_prepared_empty(L):
    assert hca_prep(L, n=127, C=None, Z=None, ws=None, out=None) == kvc.KVC_OK


def test_noalloc_rejects_before_launch(L):
    # sizes are checked before any CUDA call (fake pointers are never dereferenced)
    call = lambda **kw: L.hca_compress_noalloc(
        kw.get("C", A), A, kw.get("dt", kvc.KVC_BF16), A, 1, kw.get("n", 4096), kw.get("c", 512),
        kw.get("m", 128), A, kvc.KVC_BF16, None)
    assert call(c=2048) == kvc.KVC_ERR_TOO_LARGE
    assert call(c=1024, m=128) == kvc.KVC_ERR_TOO_LARGE
    assert call(m=400) == kvc.KVC_ERR_UNSUPPORTED
    assert call(c=12) == kvc.KVC_ERR_SHAPE
    assert call(dt=5) == kvc.KVC_ERR_DTYPE
    assert call(C=None) == kvc.KVC_ERR_NULL
    assert call(n=100, C=None) == kvc.KVC_OK  # empty: no entry, nothing touched


def test_fused_scalar_rejects_before_launch(L):
    csa = lambda **kw: L.csa_compress_fused_proj_scalar(
        kw.get("H", A), A, A, kw.get("wza", A), A, A, A, 1, kw.get("n", 4096), kw.get("d", 7168),
        kw.get("c", 512), kw.get("m", 4), kw.get("ov", 1), A, kvc.KVC_BF16, None)
    hca = lambda **kw: L.hca_compress_fused_proj_scalar(
        A, A, kw.get("wz", A), A, 1, 4096, 4096, kw.get("c", 512), kw.get("m", 128), A,
        kvc.KVC_BF16, None)
    assert csa(m=8) == kvc.KVC_ERR_UNSUPPORTED
    assert csa(ov=0) == kvc.KVC_ERR_UNSUPPORTED
    assert csa(d=100) == kvc.KVC_ERR_SHAPE
    assert csa(c=200) == kvc.KVC_ERR_SHAPE
    assert csa(wza=None) == kvc.KVC_ERR_NULL
    assert csa(wza=MIS) == kvc.KVC_ERR_ALIGN
    assert csa(n=3, H=None, wza=None) == kvc.KVC_OK  # empty
    assert hca(m=64) == kvc.KVC_ERR_UNSUPPORTED
    assert hca(wz=None) == kvc.KVC_ERR_NULL
    assert hca(wz=MIS) == kvc.KVC_ERR_ALIGN


def test_fused_empty(L):
    assert fused_csa(L, n=2, H=None, out=None) == kvc.KVC_OK
    assert fused_hca(L, batch=0, H=None, out=None) == kvc.KVC_OK


def csa_sc(L, **kw):
    a = dict(Ca=A, Cb=A, za=A, zb=A, in_dt=kvc.KVC_BF16, ba=A, bb=A, batch=1, n=1024, c=512, m=4,
             overlap=1, out=A, out_dt=kvc.KVC_BF16)
    a.update(kw)
    return L.csa_compress_scalar_logits(a["Ca"], a["Cb"], a["za"], a["zb"], a["in_dt"], a["ba"], a["bb"],
                                        a["batch"], a["n"], a["c"], a["m"], a["overlap"], a["out"],
                                        a["out_dt"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(in_dt=9), kvc.KVC_ERR_DTYPE),
    (dict(n=-1), kvc.KVC_ERR_SHAPE),
    (dict(c=12), kvc.KVC_ERR_SHAPE),
    (dict(overlap=5), kvc.KVC_ERR_SHAPE),
    (dict(za=None), kvc.KVC_ERR_NULL),
    (dict(bb=None), kvc.KVC_ERR_NULL),
    (dict(Ca=MIS), kvc.KVC_ERR_ALIGN),
    (dict(za=A + 1), kvc.KVC_ERR_ALIGN),
    (dict(in_dt=kvc.KVC_F32, za=A + 2), kvc.KVC_ERR_ALIGN),
    (dict(m=161), kvc.KVC_ERR_UNSUPPORTED),
])
def test_csa_scalar_rejects_before_launch(L, kw, status):
    assert csa_sc(L, **kw) == status


def test_scalar_logit_misc(L):
    # za may sit at any 2-byte offset for bf16 (no 16-byte rule for the logits)
    assert csa_sc(L, za=A + 2, Ca=MIS) == kvc.KVC_ERR_ALIGN  # fails on Ca, not on za
    assert csa_sc(L, overlap=0, Cb=None, zb=None, bb=None, out=MIS) == kvc.KVC_ERR_ALIGN
    assert csa_sc(L, n=2, Ca=None, za=None, out=None) == kvc.KVC_OK
    assert L.hca_compress_scalar_logits(A, None, kvc.KVC_BF16, A, 1, 256, 512, 128, A, kvc.KVC_BF16,
                                        None) == kvc.KVC_ERR_NULL
    assert L.hca_compress_scalar_logits(A, A, kvc.KVC_BF16, A, 1, 1024, 512, 400, A, kvc.KVC_BF16,
                                        None) == kvc.KVC_ERR_UNSUPPORTED
    assert L.hca_compress_scalar_logits(A, A, kvc.KVC_BF16, A, 1, 100, 512, 128, A, kvc.KVC_BF16,
                                        None) == kvc.KVC_OK


def csa_cache(L, **kw):
    a = dict(Ca=A, Cb=A, Za=A, Zb=A, in_dt=kvc.KVC_BF16, Ba=A, Bb=A, batch=1, n=1024, c=512, m=4,
             overlap=1, r=64, inv=A, ps=4.0, po=1.5, sc=1.0, nope=A, rope=A)
    a.update(kw)
    return L.csa_compress_cache(a["Ca"], a["Cb"], a["Za"], a["Zb"], a["in_dt"], a["Ba"], a["Bb"],
                                a["batch"], a["n"], a["c"], a["m"], a["overlap"], a["r"], a["inv"],
                                a["ps"], a["po"], a["sc"], a["nope"], a["rope"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(in_dt=4), kvc.KVC_ERR_DTYPE),
    (dict(r=12), kvc.KVC_ERR_SHAPE),
    (dict(r=-8), kvc.KVC_ERR_SHAPE),
    (dict(r=520), kvc.KVC_ERR_SHAPE),
    (dict(sc=float("nan")), kvc.KVC_ERR_SHAPE),
    (dict(po=float("nan")), kvc.KVC_ERR_SHAPE),
    (dict(inv=None), kvc.KVC_ERR_NULL),
    (dict(rope=None), kvc.KVC_ERR_NULL),
    (dict(nope=None), kvc.KVC_ERR_NULL),
    (dict(nope=A + 8), kvc.KVC_ERR_ALIGN),
    (dict(rope=A + 4), kvc.KVC_ERR_ALIGN),
    (dict(inv=A + 2), kvc.KVC_ERR_ALIGN),
    (dict(Ca=MIS), kvc.KVC_ERR_ALIGN),
])
def test_csa_cache_rejects_before_launch(L, kw, status):
    assert csa_cache(L, **kw) == status


def test_cache_layout_optional_parts(L):
    # r == 0: no rope part, so rope / inv_freq may be NULL (stops at the next check)
    assert csa_cache(L, r=0, rope=None, inv=None, nope=A + 8) == kvc.KVC_ERR_ALIGN
    # r == c: no nope part
    assert csa_cache(L, r=512, nope=None, rope=A + 4) == kvc.KVC_ERR_ALIGN
    assert csa_cache(L, n=3, Ca=None, nope=None) == kvc.KVC_OK  # empty problem
    assert L.hca_compress_cache(A, A, kvc.KVC_BF16, A, 1, 1024, 512, 128, 64, None, 128.0, 63.5, 1.0,
                                A, A, None) == kvc.KVC_ERR_NULL
    assert L.csa_compress_entries_cache(A, A, A, A, kvc.KVC_BF16, A, A, 1024, 512, 4, 1, A, A, A, 8,
                                        12, A, 4.0, 1.5, 1.0, A, A, None) == kvc.KVC_ERR_SHAPE
    assert L.hca_compress_entries_cache(A, A, kvc.KVC_BF16, A, 1024, 512, 128, A, A, A, 0, 64, A,
                                        128.0, 63.5, 1.0, A, A, None) == kvc.KVC_OK  # empty list


# ------------------------------------------------------------------ lightning indexer

def ix_scores(L, q=A, w=A, K=A, ks=A, nv=A, T=8, H=64, D=128, rows=1 << 20, mv=262144,
              sc=A, ld=262144):
    return L.lightning_indexer_scores(q, w, K, ks, nv, T, H, D, rows, mv, sc, ld, None)


@pytest.mark.parametrize("kw,status", [
    (dict(T=-1), kvc.KVC_ERR_SHAPE),
    (dict(rows=-1), kvc.KVC_ERR_SHAPE),
    (dict(mv=-1), kvc.KVC_ERR_SHAPE),
    (dict(ld=1000), kvc.KVC_ERR_SHAPE),            # ld < max_visible
    (dict(D=64), kvc.KVC_ERR_UNSUPPORTED),
    (dict(H=8), kvc.KVC_ERR_UNSUPPORTED),
    (dict(H=136), kvc.KVC_ERR_UNSUPPORTED),
    (dict(H=72), kvc.KVC_ERR_UNSUPPORTED),
    (dict(rows=1 << 31), kvc.KVC_ERR_UNSUPPORTED),  # TMA rows are 32-bit
    (dict(q=None), kvc.KVC_ERR_NULL),
    (dict(nv=None), kvc.KVC_ERR_NULL),
    (dict(sc=None), kvc.KVC_ERR_NULL),
    (dict(q=MIS), kvc.KVC_ERR_ALIGN),
    (dict(K=MIS), kvc.KVC_ERR_ALIGN),
    (dict(sc=A + 4), kvc.KVC_ERR_ALIGN),
    (dict(w=A + 2), kvc.KVC_ERR_ALIGN),
    (dict(ks=A + 4), kvc.KVC_ERR_ALIGN),
])
def test_indexer_scores_rejects_before_launch(L, kw, status):
    assert ix_scores(L, **kw) == status


def test_indexer_scores_empty(L):
    assert ix_scores(L, T=0, q=None, K=None) == kvc.KVC_OK
    assert ix_scores(L, mv=0, ld=0, q=None) == kvc.KVC_OK


def ix_topk(L, sc=A, ld=262144, nv=A, T=8, mv=262144, k=1024, idx=A, val=A):
    return L.indexer_topk(sc, ld, nv, T, mv, k, idx, val, None)


@pytest.mark.parametrize("kw,status", [
    (dict(k=0), kvc.KVC_ERR_SHAPE),
    (dict(k=2049), kvc.KVC_ERR_UNSUPPORTED),
    (dict(mv=327681, ld=327684), kvc.KVC_ERR_UNSUPPORTED),
    (dict(ld=262146), kvc.KVC_ERR_SHAPE),          # ld not a multiple of 4
    (dict(ld=1000), kvc.KVC_ERR_SHAPE),
    (dict(T=-1), kvc.KVC_ERR_SHAPE),
    (dict(sc=None), kvc.KVC_ERR_NULL),
    (dict(idx=None), kvc.KVC_ERR_NULL),
    (dict(sc=A + 4), kvc.KVC_ERR_ALIGN),
    (dict(nv=A + 4), kvc.KVC_ERR_ALIGN),
    (dict(idx=A + 2), kvc.KVC_ERR_ALIGN),
    (dict(val=A + 2), kvc.KVC_ERR_ALIGN),
])
def test_indexer_topk_rejects_before_launch(L, kw, status):
    assert ix_topk(L, **kw) == status


def test_indexer_topk_limits(L):
    assert L.kvc_topk_max_candidates() == 8 * 40960
    assert ix_topk(L, T=0, sc=None, idx=None) == kvc.KVC_OK


def csa_list(L, Ca=A, Cb=A, Za=A, Zb=A, in_dt=kvc.KVC_BF16, Ba=A, Bb=A, rows=4096, c=512, m=4,
             overlap=1, start=A, slen=A, entry=A, num=64, out=A, out_dt=kvc.KVC_BF16):
    return L.csa_compress_entries(Ca, Cb, Za, Zb, in_dt, Ba, Bb, rows, c, m, overlap, start, slen,
                                  entry, num, out, out_dt, None)


@pytest.mark.parametrize("kw,status", [
    (dict(in_dt=9), kvc.KVC_ERR_DTYPE),
    (dict(out_dt=3), kvc.KVC_ERR_DTYPE),
    (dict(overlap=2), kvc.KVC_ERR_SHAPE),
    (dict(rows=-1), kvc.KVC_ERR_SHAPE),
    (dict(m=0), kvc.KVC_ERR_SHAPE),
    (dict(num=-1), kvc.KVC_ERR_SHAPE),
    (dict(c=12), kvc.KVC_ERR_SHAPE),
    (dict(rows=1 << 62), kvc.KVC_ERR_SHAPE),        # rows * c * 4 bytes overflows
    (dict(num=1 << 62), kvc.KVC_ERR_SHAPE),         # num * c overflows
    (dict(start=None), kvc.KVC_ERR_NULL),
    (dict(slen=None), kvc.KVC_ERR_NULL),
    (dict(entry=None), kvc.KVC_ERR_NULL),
    (dict(Ca=None), kvc.KVC_ERR_NULL),
    (dict(Bb=None), kvc.KVC_ERR_NULL),
    (dict(out=None), kvc.KVC_ERR_NULL),
    (dict(start=A + 4), kvc.KVC_ERR_ALIGN),         # the lists are int64
    (dict(entry=A + 4), kvc.KVC_ERR_ALIGN),
    (dict(Za=MIS), kvc.KVC_ERR_ALIGN),
    (dict(Cb=MIS), kvc.KVC_ERR_ALIGN),
    (dict(Ba=A + 2), kvc.KVC_ERR_ALIGN),
    (dict(m=161), kvc.KVC_ERR_UNSUPPORTED),         # 2 m = 322 window rows
])
def test_csa_entries_rejects_before_launch(L, kw, status):
    assert csa_list(L, **kw) == status


def test_csa_entries_overlap_off_and_empty(L):
    # overlap = 0 lets the b-stream pointers be NULL (validation reaches the a-stream check)
    assert csa_list(L, overlap=0, Cb=None, Zb=None, Bb=None, Ca=MIS) == kvc.KVC_ERR_ALIGN
    # an empty list (or c == 0) is valid and reads no pointer, the lists' included
    none = dict(Ca=None, Cb=None, Za=None, Zb=None, Ba=None, Bb=None, start=None, slen=None,
                entry=None, out=None)
    assert csa_list(L, num=0, **none) == kvc.KVC_OK
    assert csa_list(L, c=0, **none) == kvc.KVC_OK


def hca_list(L, C=A, Z=A, in_dt=kvc.KVC_BF16, B=A, rows=4096, c=512, m=128, start=A, slen=A,
             entry=A, num=8, out=A, out_dt=kvc.KVC_BF16):
    return L.hca_compress_entries(C, Z, in_dt, B, rows, c, m, start, slen, entry, num, out, out_dt,
                                  None)


@pytest.mark.parametrize("kw,status", [
    (dict(in_dt=2), kvc.KVC_ERR_DTYPE),
    (dict(rows=-128), kvc.KVC_ERR_SHAPE),
    (dict(c=20), kvc.KVC_ERR_SHAPE),
    (dict(m=-1), kvc.KVC_ERR_SHAPE),
    (dict(slen=None), kvc.KVC_ERR_NULL),
    (dict(Z=None), kvc.KVC_ERR_NULL),
    (dict(B=None), kvc.KVC_ERR_NULL),
    (dict(slen=A + 4), kvc.KVC_ERR_ALIGN),
    (dict(C=MIS), kvc.KVC_ERR_ALIGN),
    (dict(out=MIS), kvc.KVC_ERR_ALIGN),
    (dict(B=A + 1), kvc.KVC_ERR_ALIGN),
    (dict(m=321), kvc.KVC_ERR_UNSUPPORTED),
])
def test_hca_entries_rejects_before_launch(L, kw, status):
    assert hca_list(L, **kw) == status


def test_hca_entries_empty(L):
    assert hca_list(L, num=0, C=None, Z=None, B=None, start=None, slen=None, entry=None,
                    out=None) == kvc.KVC_OK


def test_selftest_rejects_before_launch(L):
    assert L.kvc_selftest_bounded_wait(None, None) == kvc.KVC_ERR_NULL
    assert L.kvc_selftest_bounded_wait(A + 2, None) == kvc.KVC_ERR_ALIGN


def test_binding_raises_without_the_library(monkeypatch):
    # No CPU fallback: with libkvc.so absent every call fails loudly.
    monkeypatch.setattr(kvc, "_lib", None)
    monkeypatch.setattr(kvc, "LIB_PATH", os.path.join(ROOT, "no-such-dir", "libkvc.so"))
    with pytest.raises(RuntimeError, match="missing"):
        kvc.num_entries(8, 4)
    with pytest.raises(RuntimeError, match="missing"):
        kvc.lib()


def test_product_package_never_reaches_the_oracle():
    # The oracle is test infrastructure: the package neither imports it nor names it in an
    # import, and importing the package (and its binding) loads no module of it.
    pkg = os.path.join(ROOT, "kv_token_compressor_b200")
    for name in sorted(os.listdir(pkg)):
        if name.endswith(".py"):
            src = open(os.path.join(pkg, name)).read()
            assert not re.search(r"^\s*(from|import)\s+oracle\b", src, re.M), name
    code = ("import sys; import kv_token_compressor_b200, kv_token_compressor_b200.kvc, "
            "kv_token_compressor_b200.synth, kv_token_compressor_b200.shard; "
            "print(sorted(m for m in sys.modules if m == 'oracle' or m.startswith('oracle.')))")
    out = subprocess.run([sys.executable, "-c", code], cwd=ROOT, capture_output=True,
                         text=True, timeout=300)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "[]"


def _header_prototypes():
    """name -> (return type, [parameter types]) for every KVC_API declaration, with the
    comments removed and the parameter names dropped."""
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", " ", src)
    protos = {}
    for ret, name, params in re.findall(r"KVC_API\s+([\w\s\*]+?)\s*\b(\w+)\s*\(([^)]*)\)\s*;", src):
        types = []
        for p in params.split(","):
            p = " ".join(p.split())
            if not p or p == "void":
                continue
            p = re.sub(r"\b\w+$", "", p).strip()  # drop the parameter name
            types.append(p.replace(" *", "*"))
        protos[name] = (" ".join(ret.split()).replace(" *", "*"), types)
    return protos


# The ctypes class each C type of the header must be bound with (pointers of any kind
# travel as void*; enums are C ints).
_CTYPE = {
    "int64_t": ctypes.c_int64, "int32_t": ctypes.c_int32, "double": ctypes.c_double,
    "float": ctypes.c_float, "kvc_status": ctypes.c_int, "kvc_dtype": ctypes.c_int,
    "kvc_stream": ctypes.c_void_p, "const char*": ctypes.c_char_p, "void": None,
}


def _ctype_of(t):
    if t.endswith("*") and t != "const char*":
        return ctypes.c_void_p
    return _CTYPE[t]


def test_binding_signatures_match_the_header():
    protos = _header_prototypes()
    assert set(protos) == set(header_entry_points())
    assert set(kvc.SIGNATURES) == set(protos)
    for name, (ret, params) in protos.items():
        res, args = kvc.SIGNATURES[name]
        assert res is _ctype_of(ret), (name, ret)
        assert len(args) == len(params), (name, len(args), len(params))
        for i, (a, p) in enumerate(zip(args, params)):
            assert a is _ctype_of(p), (name, i, p, a)


# ---- the Python binding refuses tensors the library would misread (checked before any
# pointer is taken, so CPU tensors exercise it: a consistent call gets as far as the
# "must be on a CUDA device" check)

def _z(*shape, dt="f32"):
    import torch

    return torch.zeros(shape, dtype={"f32": torch.float32, "bf16": torch.bfloat16,
                                     "f64": torch.float64, "i64": torch.int64}[dt])


def _csa_args(**kw):
    a = dict(Ca=_z(1, 64, 64, dt="bf16"), Cb=_z(1, 64, 64, dt="bf16"), Za=_z(1, 64, 64, dt="bf16"),
             Zb=_z(1, 64, 64, dt="bf16"), Ba=_z(4, 64), Bb=_z(4, 64))
    a.update(kw)
    return a


def _entries_args(**kw):
    a = dict(Ca=_z(64, 64), Cb=_z(64, 64), Za=_z(64, 64), Zb=_z(64, 64), Ba=_z(4, 64), Bb=_z(4, 64),
             seq_start=_z(2, dt="i64"), seq_len=_z(2, dt="i64"), entry=_z(2, dt="i64"))
    a.update(kw)
    return a


BINDING_CASES = [
    ("csa short Za", lambda: kvc.csa_compress(**_csa_args(Za=_z(1, 32, 64, dt="bf16"))), "Za holds"),
    ("csa Zb dtype", lambda: kvc.csa_compress(**_csa_args(Zb=_z(1, 64, 64))), "Zb must be"),
    ("csa Cb dtype", lambda: kvc.csa_compress(**_csa_args(Cb=_z(1, 64, 64))), "Cb must be"),
    ("csa bias width", lambda: kvc.csa_compress(**_csa_args(Ba=_z(4, 32))), "Ba holds"),
    ("csa bias dtype", lambda: kvc.csa_compress(**_csa_args(Bb=_z(4, 64, dt="bf16"))), "Bb must be"),
    ("csa consistent", lambda: kvc.csa_compress(**_csa_args()), "CUDA device"),
    ("csa overlap off", lambda: kvc.csa_compress(**_csa_args(Cb=None, Zb=None, Bb=_z(1)),
                                                 overlap=False), "CUDA device"),
    ("hca bias rows", lambda: kvc.hca_compress(_z(1, 256, 64), _z(1, 256, 64), _z(64, 64), m=128),
     "B holds"),
    ("hca Z dtype", lambda: kvc.hca_compress(_z(1, 256, 64), _z(1, 256, 64, dt="f64"),
                                             _z(128, 64), m=128), "Z must be"),
    ("scalar zb size", lambda: kvc.csa_compress_scalar_logits(
        _z(1, 64, 64), _z(1, 64, 64), _z(1, 64), _z(1, 32), _z(4), _z(4)), "zb holds"),
    ("scalar bias", lambda: kvc.hca_compress_scalar_logits(_z(1, 256, 64), _z(1, 256), _z(64),
                                                           m=128), "b holds"),
    ("entries Za", lambda: kvc.csa_compress_entries(**_entries_args(Za=_z(63, 64))), "Za holds"),
    ("entries consistent", lambda: kvc.csa_compress_entries(**_entries_args()), "CUDA device"),
    ("hca entries B", lambda: kvc.hca_compress_entries(
        _z(256, 64), _z(256, 64), _z(128, 64, dt="f64"), _z(1, dt="i64"), _z(1, dt="i64"),
        _z(1, dt="i64")), "B must be"),
    ("cache inv_freq", lambda: kvc.csa_compress_cache(**_csa_args(), r=16, inv_freq=_z(4)),
     "inv_freq holds"),
    ("cache bad r reaches the library", lambda: kvc.csa_compress_cache(
        **_csa_args(), r=12, inv_freq=_z(4)), "CUDA device"),
    ("fused H dtype", lambda: kvc.hca_compress_fused_proj(
        _z(256, 128), _z(128, 128, dt="bf16"), _z(128, 128, dt="bf16"), _z(128, 128), 1, 256),
     "H must be"),
    ("fused short H", lambda: kvc.hca_compress_fused_proj(
        _z(255, 128, dt="bf16"), _z(128, 128, dt="bf16"), _z(128, 128, dt="bf16"), _z(128, 128),
        1, 256), "H holds"),
    ("fused W_zb", lambda: kvc.csa_compress_fused_proj(
        _z(64, 128, dt="bf16"), *[_z(128, 128, dt="bf16")] * 3, _z(64, 128, dt="bf16"),
        _z(4, 128), _z(4, 128), 1, 64), "W_zb holds"),
    ("indexer K width", lambda: kvc.lightning_indexer_scores(
        _z(2, 4, 128, dt="bf16"), _z(2, 4), _z(100, 64, dt="bf16"), _z(2, dt="i64"),
        _z(2, dt="i64"), 100), "K must be"),
    ("indexer w dtype", lambda: kvc.lightning_indexer_scores(
        _z(2, 4, 128, dt="bf16"), _z(2, 4, dt="f64"), _z(100, 128, dt="bf16"), _z(2, dt="i64"),
        _z(2, dt="i64"), 100), "w must be"),
    ("topk scores dtype", lambda: kvc.indexer_topk(_z(2, 8, dt="f64"), _z(2, dt="i64"), 4, 8),
     "scores must be"),
]


@pytest.mark.parametrize("name,call,msg", BINDING_CASES, ids=[c[0] for c in BINDING_CASES])
def test_binding_refuses_tensors_the_library_would_misread(L, name, call, msg):
    with pytest.raises(ValueError, match=msg):
        call()


C_CONSUMER = r"""
#include <stdio.h>
#include <stddef.h>
#include "kvc.h"

/* A plain C99 program against the C ABI.  Only calls that fail validation before any CUDA
 * call are made, so it runs without a GPU. */
int main(void) {
  int bad = 0;
  if (kvc_num_entries(1 << 20, 4) != 262144 || kvc_num_entries(1 << 20, 128) != 8192) bad |= 1;
  if (kvc_num_entries(-1, 4) != -1) bad |= 2;
  if (csa_compress(NULL, NULL, NULL, NULL, KVC_BF16, NULL, NULL, 1, 1024, 512, 4, 1, NULL,
                   KVC_BF16, NULL) != KVC_ERR_NULL) bad |= 4;
  if (hca_compress(NULL, NULL, KVC_BF16, NULL, 1, 1024, 512, 128, NULL, KVC_BF16, NULL)
      != KVC_ERR_NULL) bad |= 8;
  /* an empty problem is valid and touches nothing */
  if (csa_compress(NULL, NULL, NULL, NULL, KVC_BF16, NULL, NULL, 0, 1024, 512, 4, 1, NULL,
                   KVC_BF16, NULL) != KVC_OK) bad |= 16;
  if (kvc_selftest_bounded_wait(NULL, NULL) != KVC_ERR_NULL) bad |= 32;
  if (kvc_status_string(KVC_ERR_TIMEOUT) == NULL) bad |= 64;
  if (kvc_topk_max_candidates() <= 0) bad |= 128;
  /* nothing was launched: the record of the last kernel is still empty */
  if (kvc_last_kernel() == NULL || kvc_last_kernel()[0] != '\0') bad |= 256;
  printf("%s %d\n", kvc_status_string(KVC_ERR_SHAPE), bad);
  return bad;
}
"""


def test_plain_c_program_uses_the_abi(L, tmp_path):
    # The header compiles as C99 (no C++ or CUDA types leak into it) and a C program linked
    # against libkvc.so gets the documented statuses.
    src = tmp_path / "consumer.c"
    src.write_text(C_CONSUMER)
    exe = tmp_path / "consumer"
    lib_dir = os.path.dirname(kvc.LIB_PATH)
    cc = subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-pedantic", "-I",
                         os.path.join(ROOT, "include"), str(src), "-L", lib_dir, "-lkvc",
                         "-Wl,-rpath," + lib_dir, "-o", str(exe)], capture_output=True, text=True)
    assert cc.returncode == 0, cc.stderr
    run = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert run.returncode == 0, (run.returncode, run.stdout, run.stderr)
    assert run.stdout.split()[-1] == "0"


def test_sync_check_setting_round_trips():
    """kvc_set_sync_check / kvc_sync_check: off by default, any nonzero is on."""
    L = kvc.lib()
    assert L.kvc_sync_check() == 0
    try:
        L.kvc_set_sync_check(7)
        assert L.kvc_sync_check() == 1 and kvc.sync_check()
        kvc.set_sync_check(False)
        assert L.kvc_sync_check() == 0 and not kvc.sync_check()
    finally:
        L.kvc_set_sync_check(0)
