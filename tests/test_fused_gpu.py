"""GPU parity of the fused projection + pool path (tcgen05 GEMM with the softmax-pool in
its epilogue) through the C ABI, against the fp64 oracle on the same seeded inputs."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from gpu_util import check_close, host64, tdtype
from kv_token_compressor_b200 import kvc, synth
from oracle import compressor as O

pytestmark = pytest.mark.gpu


def _dev(d):
    out = {}
    for k, v in d.items():
        t = torch.from_numpy(np.ascontiguousarray(v)).cuda()
        out[k] = t if k.startswith("B") else t.to(torch.bfloat16)
    return out


CSA_CASES = [
    # batch, n, d, c   (m = 4, overlap)
    (1, 1024, 128, 128),
    (1, 1000, 256, 256),
    (3, 517, 192, 128),
    (2, 4 * 700 + 2, 64, 384),
    (1, 36, 512, 128),
    # every entry of several pieces and 256-row tiles (shortened last tiles), 4 groups
    (2, 4 * 2000 + 3, 256, 512),
]


@pytest.mark.parametrize("out_dt", ["bf16", "f32"])
@pytest.mark.parametrize("batch,n,d,c", CSA_CASES)
def test_csa_fused_small(batch, n, d, c, out_dt):
    h = synth.fused_inputs("csa", batch, n, d, c, 4, seed=n + d + c)
    t = _dev(h)
    out = kvc.csa_compress_fused_proj(t["H"], t["W_kva"], t["W_kvb"], t["W_za"], t["W_zb"], t["Ba"],
                                      t["Bb"], batch, n, m=4, out_dtype=tdtype(out_dt))
    torch.cuda.synchronize()
    assert kvc.device_status() == kvc.KVC_OK
    ref = O.csa_compress_fused(h["H"], h["W_kva"], h["W_kvb"], h["W_za"], h["W_zb"], h["Ba"],
                               h["Bb"], batch, n, 4, True)
    assert out.shape == (batch, n // 4, c)
    check_close(out, ref, out_dt, f"csa fused {batch}x{n} d={d} c={c}")


HCA_CASES = [
    (1, 128 * 4, 128, 128),
    (2, 128 * 5 + 17, 256, 256),
    (3, 128 * 3, 64, 384),
    (1, 128 * 40, 448, 128),
    # channel groups in pairs over a CTA pair; an odd entry count ends in a half tile
    (2, 128 * 9 + 5, 128, 512),
]


@pytest.mark.parametrize("out_dt", ["bf16", "f32"])
@pytest.mark.parametrize("batch,n,d,c", HCA_CASES)
def test_hca_fused_small(batch, n, d, c, out_dt):
    h = synth.fused_inputs("hca", batch, n, d, c, 128, seed=3 + n + d + c)
    t = _dev(h)
    out = kvc.hca_compress_fused_proj(t["H"], t["W_kv"], t["W_z"], t["B"], batch, n, m=128,
                                      out_dtype=tdtype(out_dt))
    torch.cuda.synchronize()
    assert kvc.device_status() == kvc.KVC_OK
    ref = O.hca_compress_fused(h["H"], h["W_kv"], h["W_z"], h["B"], batch, n, 128)
    assert out.shape == (batch, n // 128, c)
    check_close(out, ref, out_dt, f"hca fused {batch}x{n} d={d} c={c}")


@pytest.mark.parametrize("seed", range(4))
def test_fused_random_shapes(seed):
    """Seeded random fused problems: d a multiple of 64 up to 640, c a multiple of 128 up to
    768, ragged n (CSA m = 4 with overlap, HCA m' = 128), 1-3 sequences, both output types;
    each output between canary bands that must come back untouched."""
    rng = np.random.default_rng(900 + seed)
    for mode in ("csa", "hca"):
        batch = int(rng.integers(1, 4))
        d = 64 * int(rng.integers(1, 11))
        c = 128 * int(rng.integers(1, 7))
        m = 4 if mode == "csa" else 128
        n = int(rng.integers(m, 3000 if mode == "csa" else 6000))
        out_dt = rng.choice(["bf16", "f32"])
        h = synth.fused_inputs(mode, batch, n, d, c, m, seed=seed * 31 + d + c)
        t = _dev(h)
        ne = n // m
        buf = torch.full((batch * ne * c + 128,), -555.0, device="cuda", dtype=tdtype(out_dt))
        out = buf[64:64 + batch * ne * c].view(batch, ne, c)
        if mode == "csa":
            kvc.csa_compress_fused_proj(t["H"], t["W_kva"], t["W_kvb"], t["W_za"], t["W_zb"],
                                        t["Ba"], t["Bb"], batch, n, m=4, out=out,
                                        out_dtype=tdtype(out_dt))
            ref = O.csa_compress_fused(h["H"], h["W_kva"], h["W_kvb"], h["W_za"], h["W_zb"],
                                       h["Ba"], h["Bb"], batch, n, 4, True)
        else:
            kvc.hca_compress_fused_proj(t["H"], t["W_kv"], t["W_z"], t["B"], batch, n, m=128,
                                        out=out, out_dtype=tdtype(out_dt))
            ref = O.hca_compress_fused(h["H"], h["W_kv"], h["W_z"], h["B"], batch, n, 128)
        what = f"{mode} fused b={batch} n={n} d={d} c={c} {out_dt} ({kvc.last_kernel()})"
        assert kvc.device_status() == kvc.KVC_OK, what
        check_close(out, ref, out_dt, what)
        assert bool(torch.all(buf[:64] == -555.0)) and bool(torch.all(buf[64 + batch * ne * c:] == -555.0)), what


def test_fused_matches_streaming_on_identity():
    """d = c and W = scaled identities: the fused streams are exactly (scaled) H, so the
    fused path must agree with the streaming kernel fed those streams."""
    n, c = 512, 128
    rng = np.random.default_rng(0)
    H = synth.round_to_bf16(rng.standard_normal((n, c), dtype=np.float32))
    I = np.eye(c, dtype=np.float32)
    Ht = torch.from_numpy(H).cuda().to(torch.bfloat16)
    Wi = {k: torch.from_numpy(s * I).cuda().to(torch.bfloat16)
          for k, s in (("kva", 1.0), ("kvb", -2.0), ("za", 0.5), ("zb", 2.0))}
    Ba = torch.from_numpy((0.3 * rng.standard_normal((4, c))).astype(np.float32)).cuda()
    Bb = torch.from_numpy((0.3 * rng.standard_normal((4, c))).astype(np.float32)).cuda()
    fused = kvc.csa_compress_fused_proj(Ht, Wi["kva"], Wi["kvb"], Wi["za"], Wi["zb"], Ba, Bb, 1, n,
                                        out_dtype=torch.float32)
    S = Ht[None]
    streamed = kvc.csa_compress(S, (-2.0 * S.float()).to(torch.bfloat16), (0.5 * S.float()).to(torch.bfloat16),
                                (2.0 * S.float()).to(torch.bfloat16), Ba, Bb, m=4, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.max(torch.abs(fused - streamed)).item() <= 1e-5 * torch.max(torch.abs(streamed)).item()


# ------------------------------------------------------------------ full size, sampled

def _sampled_check(mode, w, ents_per_seq, seed):
    t = synth.fused_inputs_torch(mode, w["batch"], w["n"], w["d"], w["c"], w["m"], seed=seed)
    batch, n, m = w["batch"], w["n"], w["m"]
    if mode == "csa":
        out = kvc.csa_compress_fused_proj(t["H"], t["W_kva"], t["W_kvb"], t["W_za"], t["W_zb"],
                                          t["Ba"], t["Bb"], batch, n, m=4, out_dtype=torch.bfloat16)
    else:
        out = kvc.hca_compress_fused_proj(t["H"], t["W_kv"], t["W_z"], t["B"], batch, n, m=128,
                                          out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert kvc.device_status() == kvc.KVC_OK
    ne = n // m
    assert out.shape == (batch, ne, w["c"])
    assert torch.isfinite(out.float()).all().item()
    rng = np.random.default_rng(seed)
    entries = []
    for b in range(batch):
        pick = set(rng.choice(ne, size=min(ents_per_seq, ne), replace=False).tolist())
        pick |= {0, 1, ne - 1}
        # tile boundaries (32 and 64 entries per tile) and piece boundaries
        pick |= {min(ne - 1, 32 * k + d) for k in range(1, 9) for d in (-1, 0, 1)}
        pick |= {min(ne - 1, (ne * r) // P + d) for P in (18, 37, 74) for r in range(1, 4)
                 for d in (-1, 0, 1)}
        entries += [(b, i) for i in sorted(pick)]
    Ws = {k: host64(v) for k, v in t.items() if k.startswith("W") or k.startswith("B")}
    refs, got = [], []
    for b, i in entries:
        lo = m * (i - 1) if (mode == "csa" and i > 0) else m * i
        hi = m * (i + 1)
        rows = host64(t["H"][b * n + lo:b * n + hi])
        # a mini "sequence" holding just the rows entry i reads
        if mode == "csa":
            j = 1 if i > 0 else 0
            r = O.csa_compress_fused(rows, Ws["W_kva"], Ws["W_kvb"], Ws["W_za"], Ws["W_zb"], Ws["Ba"],
                                     Ws["Bb"], 1, hi - lo, 4, True, entries=[(0, j)])[0]
        else:
            r = O.hca_compress_fused(rows, Ws["W_kv"], Ws["W_z"], Ws["B"], 1, m, 128)[0, 0]
        refs.append(r)
        got.append(host64(out[b, i]))
    check_close(torch.from_numpy(np.array(got)), np.array(refs), "bf16", f"{mode} fused full sampled")


def test_csa_fused_n32768_d7168_sampled():
    _sampled_check("csa", synth.WORKLOADS["csa_fused_n32768_d7168"], 150, 0)


def test_hca_fused_4x131072_d4096_sampled():
    _sampled_check("hca", synth.WORKLOADS["hca_fused_4x131072_d4096"], 40, 0)
    torch.cuda.empty_cache()


def test_fused_unsupported_m_reports():
    x = torch.zeros((64, 128), device="cuda", dtype=torch.bfloat16)
    w = torch.zeros((128, 128), device="cuda", dtype=torch.bfloat16)
    b = torch.zeros((8, 128), device="cuda")
    with pytest.raises(kvc.KvcError) as e:
        kvc.csa_compress_fused_proj(x, w, w, w, w, b, b, 1, 64, m=8)
    assert e.value.status == kvc.KVC_ERR_UNSUPPORTED
