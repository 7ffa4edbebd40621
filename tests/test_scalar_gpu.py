"""GPU parity of the scalar-logit compressor (one logit per token and stream, a scalar
weight per window row) through the C ABI, against the fp64 oracle."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from gpu_util import check_close, dev, host64, tdtype
from kv_token_compressor_b200 import kvc, synth
from oracle import compressor as O

pytestmark = pytest.mark.gpu


def _csa(d, m, overlap, in_dt, out_dt):
    t = {k: dev(v, in_dt) if k in ("Ca", "Cb", "za", "zb") else dev(v, "f32") for k, v in d.items()}
    out = kvc.csa_compress_scalar_logits(t["Ca"], t["Cb"], t["za"], t["zb"], t["ba"], t["bb"], m=m,
                                         overlap=overlap, out_dtype=tdtype(out_dt))
    torch.cuda.synchronize()
    return out


CSA_CASES = [
    (1, 1024, 512, 4, True),
    (3, 4 * 37 + 3, 136, 4, True),
    (2, 50, 24, 1, True),
    (2, 8 * 21 + 5, 72, 8, True),
    (2, 4 * 33 + 1, 520, 4, False),
    (1, 160 * 2, 264, 160, True),
]


@pytest.mark.parametrize("in_dt,out_dt", [("f32", "f32"), ("bf16", "bf16"), ("bf16", "f32"),
                                          ("f32", "bf16")])
@pytest.mark.parametrize("batch,n,c,m,overlap", CSA_CASES)
def test_csa_scalar_shapes(batch, n, c, m, overlap, in_dt, out_dt):
    d = synth.scalar_inputs("csa", batch, n, c, m, in_dt, seed=n + c + m)
    out = _csa(d, m, overlap, in_dt, out_dt)
    ref = O.csa_compress_scalar(d["Ca"], d["Cb"] if overlap else None, d["za"],
                                d["zb"] if overlap else None, d["ba"], d["bb"] if overlap else None,
                                m, overlap)
    assert out.shape == (batch, n // m, c)
    check_close(out, ref, out_dt, f"csa scalar {batch}x{n}x{c} m={m}")


HCA_CASES = [(1, 65536, 512, 128), (2, 128 * 5 + 17, 520, 128), (3, 64 * 7, 24, 64),
             (1, 320 * 2, 16, 320), (1, 40, 8, 1)]


@pytest.mark.parametrize("in_dt,out_dt", [("f32", "f32"), ("bf16", "bf16")])
@pytest.mark.parametrize("batch,n,c,m", HCA_CASES)
def test_hca_scalar_shapes(batch, n, c, m, in_dt, out_dt):
    d = synth.scalar_inputs("hca", batch, n, c, m, in_dt, seed=3 + n + c + m)
    out = kvc.hca_compress_scalar_logits(dev(d["C"], in_dt), dev(d["z"], in_dt), dev(d["b"], "f32"),
                                         m=m, out_dtype=tdtype(out_dt))
    torch.cuda.synchronize()
    ref = O.hca_compress_scalar(d["C"], d["z"], d["b"], m)
    assert out.shape == (batch, n // m, c)
    check_close(out, ref, out_dt, f"hca scalar {batch}x{n}x{c} m={m}")


def test_scalar_matches_per_channel_kernel():
    """Scalar logits broadcast over channels through the per-channel kernel give the same
    entries (both fp32; the weights agree up to exp2 rounding)."""
    d = synth.scalar_inputs("csa", 2, 4 * 200, 256, 4, "f32", seed=9)
    sc = _csa(d, 4, True, "f32", "f32")
    rep = lambda z: np.ascontiguousarray(np.repeat(z[..., None], 256, axis=-1))
    pc = kvc.csa_compress(dev(d["Ca"], "f32"), dev(d["Cb"], "f32"), dev(rep(d["za"]), "f32"),
                          dev(rep(d["zb"]), "f32"), dev(rep(d["ba"]), "f32"), dev(rep(d["bb"]), "f32"),
                          m=4, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.max(torch.abs(sc - pc)).item() <= 1e-5 * torch.max(torch.abs(pc)).item()


def test_scalar_long_sampled():
    """n = 2^20, c = 512, bf16: sampled entries against the oracle one by one."""
    n = 1 << 20
    t = synth.scalar_inputs_torch("csa", 1, n, 512, 4, "bf16", seed=0)
    out = kvc.csa_compress_scalar_logits(t["Ca"], t["Cb"], t["za"], t["zb"], t["ba"], t["bb"], m=4)
    torch.cuda.synchronize()
    ne = n // 4
    rng = np.random.default_rng(0)
    ents = sorted(set(rng.choice(ne, 300, replace=False).tolist()) | {0, 1, ne - 1})
    ba, bb = host64(t["ba"]), host64(t["bb"])
    refs, got = [], []
    for i in ents:
        lo = 4 * (i - 1) if i > 0 else 0
        sl = slice(lo, 4 * i + 4)
        mini = {k: t[k][:, sl].float().cpu().numpy() for k in ("Ca", "Cb", "za", "zb")}
        j = 1 if i > 0 else 0
        refs.append(O.csa_compress_scalar(mini["Ca"], mini["Cb"], mini["za"], mini["zb"], ba, bb, 4,
                                          True, entries=[(0, j)])[0])
        got.append(host64(out[0, i]))
    check_close(torch.from_numpy(np.array(got)), np.array(refs), "bf16", "csa scalar n=2^20")


@pytest.mark.parametrize("seed", range(4))
def test_scalar_random_shapes(seed):
    """Seeded random scalar-logit problems: CSA with m in {1, 2, 4, 8, 12} (with and
    without overlap) and HCA with m in {8, 32, 128, 200}; c any multiple of 8 up to 1024,
    ragged n, 1-3 sequences, every input/output dtype pair; outputs between canary bands."""
    rng = np.random.default_rng(300 + seed)
    for mode in ("csa", "hca"):
        batch = int(rng.integers(1, 4))
        c = 8 * int(rng.integers(1, 129))
        in_dt, out_dt = rng.choice(["bf16", "f32"]), rng.choice(["bf16", "f32"])
        m = int(rng.choice([1, 2, 4, 8, 12] if mode == "csa" else [8, 32, 128, 200]))
        n = int(rng.integers(m, min(40 * m + 5, 2_000_000 // c)))
        d = synth.scalar_inputs(mode, batch, n, c, m, in_dt, seed=seed * 7 + m)
        ne = n // m
        buf = torch.full((batch * ne * c + 128,), -333.0, device="cuda", dtype=tdtype(out_dt))
        out = buf[64:64 + batch * ne * c].view(batch, ne, c)
        if mode == "csa":
            overlap = bool(rng.random() < 0.7)
            t = {k: dev(v, in_dt) if k in ("Ca", "Cb", "za", "zb") else dev(v, "f32") for k, v in d.items()}
            kvc.csa_compress_scalar_logits(t["Ca"], t["Cb"], t["za"], t["zb"], t["ba"], t["bb"], m=m,
                                           overlap=overlap, out=out, out_dtype=tdtype(out_dt))
            ref = O.csa_compress_scalar(d["Ca"], d["Cb"] if overlap else None, d["za"],
                                        d["zb"] if overlap else None, d["ba"],
                                        d["bb"] if overlap else None, m, overlap)
        else:
            kvc.hca_compress_scalar_logits(dev(d["C"], in_dt), dev(d["z"], in_dt), dev(d["b"], "f32"),
                                           m=m, out=out, out_dtype=tdtype(out_dt))
            ref = O.hca_compress_scalar(d["C"], d["z"], d["b"], m)
        what = f"{mode} scalar b={batch} n={n} c={c} m={m} {in_dt}->{out_dt} ({kvc.last_kernel()})"
        assert kvc.device_status() == kvc.KVC_OK, what
        check_close(out, ref, out_dt, what)
        assert bool(torch.all(buf[:64] == -333.0)) and bool(torch.all(buf[64 + batch * ne * c:] == -333.0)), what
