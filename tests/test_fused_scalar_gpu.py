"""GPU parity of the fused scalar-logit compressors (csa/hca_compress_fused_proj_scalar:
value streams on the tensor cores, one score per token and stream beside them) against the
fp64 oracle: the streams and scores projected in float64 (oracle.project), then the
scalar-logit pool (oracle.csa_compress_scalar / hca_compress_scalar).  Outputs are written
between canary bands that must come back untouched."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from gpu_util import check_close, host64, tdtype
from kv_token_compressor_b200 import kvc, synth
from oracle import compressor as O

pytestmark = pytest.mark.gpu

GUARD, CANARY = 64, -1280.0


def _dev(h):
    return {k: torch.from_numpy(np.ascontiguousarray(v)).cuda().to(
        torch.float32 if k.startswith("b") else torch.bfloat16) for k, v in h.items()}


def _guarded(shape, dtype):
    numel = int(np.prod(shape))
    buf = torch.full((numel + 2 * GUARD,), CANARY, dtype=dtype, device="cuda")
    return buf, buf[GUARD:GUARD + numel].view(shape)


def _guards_ok(buf, numel):
    return bool(torch.all(buf[:GUARD] == CANARY)) and bool(torch.all(buf[GUARD + numel:] == CANARY))


def _streams(h, batch, n, names):
    """fp64 projections: values [batch, n, c], scores [batch, n]."""
    out = {}
    for k in names:
        w = h[k]
        p = O.project(h["H"], w if w.ndim == 2 else w[:, None])
        out[k] = p.reshape(batch, n, -1) if w.ndim == 2 else p.reshape(batch, n)
    return out


CSA_CASES = [
    # batch, n, d, c
    (1, 1024, 128, 128),
    (2, 4 * 700 + 2, 128, 512),   # several tiles and pieces per sequence, carried partials
    (3, 517, 192, 256),
    (1, 36, 512, 128),
    (2, 4 * 2000 + 3, 64, 384),   # an odd number of channel groups: the last pair is half empty
]


@pytest.mark.parametrize("out_dt", ["bf16", "f32"])
@pytest.mark.parametrize("batch,n,d,c", CSA_CASES)
def test_csa_fused_scalar(batch, n, d, c, out_dt):
    h = synth.fused_scalar_inputs("csa", batch, n, d, c, 4, seed=n + d + c)
    t = _dev(h)
    buf, out = _guarded((batch, n // 4, c), tdtype(out_dt))
    kvc.csa_compress_fused_proj_scalar(t["H"], t["W_kva"], t["W_kvb"], t["w_za"], t["w_zb"],
                                       t["ba"], t["bb"], batch, n, out=out, out_dtype=tdtype(out_dt))
    assert kvc.last_kernel() == "fused_scalar_kernel/csa"
    assert kvc.device_status() == kvc.KVC_OK
    s = _streams(h, batch, n, ("W_kva", "W_kvb", "w_za", "w_zb"))
    ref = O.csa_compress_scalar(s["W_kva"], s["W_kvb"], s["w_za"], s["w_zb"], h["ba"], h["bb"], 4,
                                True)
    check_close(out, ref, out_dt, f"csa fused scalar {batch}x{n} d={d} c={c}")
    assert _guards_ok(buf, out.numel())


HCA_CASES = [
    (1, 128 * 4, 128, 128),       # one channel group: three of the quad's four are empty
    (2, 128 * 5 + 17, 256, 256),
    (3, 128 * 3, 64, 384),
    (2, 128 * 9 + 5, 128, 512),   # an odd window count: the last tile holds one window
    (1, 128 * 40, 448, 1024),
]


@pytest.mark.parametrize("out_dt", ["bf16", "f32"])
@pytest.mark.parametrize("batch,n,d,c", HCA_CASES)
def test_hca_fused_scalar(batch, n, d, c, out_dt):
    h = synth.fused_scalar_inputs("hca", batch, n, d, c, 128, seed=3 + n + d + c)
    t = _dev(h)
    buf, out = _guarded((batch, n // 128, c), tdtype(out_dt))
    kvc.hca_compress_fused_proj_scalar(t["H"], t["W_kv"], t["w_z"], t["b"], batch, n, out=out,
                                       out_dtype=tdtype(out_dt))
    assert kvc.last_kernel() == "fused_scalar_kernel/hca"
    assert kvc.device_status() == kvc.KVC_OK
    s = _streams(h, batch, n, ("W_kv", "w_z"))
    ref = O.hca_compress_scalar(s["W_kv"], s["w_z"], h["b"], 128)
    check_close(out, ref, out_dt, f"hca fused scalar {batch}x{n} d={d} c={c}")
    assert _guards_ok(buf, out.numel())


def test_fused_scalar_matches_streamed_scalar():
    """The fused form against the streaming scalar-logit kernel fed streams the GPU
    projected (fp32 GEMM, then rounded to fp32 streams): the two agree to fp32 accuracy."""
    batch, n, d, c = 2, 4 * 500, 256, 256
    t = synth.fused_scalar_inputs_torch("csa", batch, n, d, c, 4, seed=7)
    fused = kvc.csa_compress_fused_proj_scalar(t["H"], t["W_kva"], t["W_kvb"], t["w_za"], t["w_zb"],
                                               t["ba"], t["bb"], batch, n, out_dtype=torch.float32)
    Hf = t["H"].float()
    Ca = (Hf @ t["W_kva"].float()).view(batch, n, c)
    Cb = (Hf @ t["W_kvb"].float()).view(batch, n, c)
    za = (Hf @ t["w_za"].float()).view(batch, n)
    zb = (Hf @ t["w_zb"].float()).view(batch, n)
    streamed = kvc.csa_compress_scalar_logits(Ca, Cb, za, zb, t["ba"], t["bb"], m=4,
                                              out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert kvc.device_status() == kvc.KVC_OK
    scale = torch.max(torch.abs(streamed)).item()
    assert torch.max(torch.abs(fused - streamed)).item() <= 1e-4 * scale


@pytest.mark.parametrize("mode", ["csa", "hca"])
def test_fused_scalar_full_size_sampled(mode):
    """The fused workloads' shapes (CSA: H [32768, 7168], c = 512; HCA: 4 x 131072 tokens,
    d = 4096) in the scalar form: sampled entries (random, first and last, tile and piece
    boundaries) against the oracle evaluated on the rows each entry reads."""
    w = synth.WORKLOADS["csa_fused_n32768_d7168" if mode == "csa" else "hca_fused_4x131072_d4096"]
    batch, n, d, c, m = w["batch"], w["n"], w["d"], w["c"], w["m"]
    t = synth.fused_scalar_inputs_torch(mode, batch, n, d, c, m, seed=1)
    if mode == "csa":
        out = kvc.csa_compress_fused_proj_scalar(t["H"], t["W_kva"], t["W_kvb"], t["w_za"],
                                                 t["w_zb"], t["ba"], t["bb"], batch, n)
    else:
        out = kvc.hca_compress_fused_proj_scalar(t["H"], t["W_kv"], t["w_z"], t["b"], batch, n)
    assert kvc.device_status() == kvc.KVC_OK
    ne = n // m
    rng = np.random.default_rng(2)
    h = {k: host64(v) for k, v in t.items() if k != "H"}
    got, refs = [], []
    for b in range(batch):
        pick = set(rng.choice(ne, size=min(60 if mode == "csa" else 12, ne), replace=False).tolist())
        pick |= {0, 1, ne - 1} | {min(ne - 1, 64 * k + dd) for k in range(1, 8) for dd in (-1, 0, 1)}
        for i in sorted(pick):
            lo = m * (i - 1) if (mode == "csa" and i > 0) else m * i
            rows = host64(t["H"][b * n + lo:b * n + m * (i + 1)])
            proj = lambda k: O.project(rows, h[k] if h[k].ndim == 2 else h[k][:, None])
            if mode == "csa":
                j = 1 if i > 0 else 0
                r = O.csa_compress_scalar(proj("W_kva")[None], proj("W_kvb")[None],
                                          proj("w_za")[None, :, 0], proj("w_zb")[None, :, 0],
                                          h["ba"], h["bb"], 4, True, entries=[(0, j)])[0]
            else:
                r = O.hca_compress_scalar(proj("W_kv")[None], proj("w_z")[None, :, 0], h["b"],
                                          128)[0, 0]
            refs.append(r)
            got.append(host64(out[b, i]))
    check_close(torch.from_numpy(np.array(got)), np.array(refs), "bf16", f"{mode} fused scalar sampled")
    del t
    torch.cuda.empty_cache()


def test_fused_scalar_refuses_other_windows():
    x = torch.zeros((64, 128), device="cuda", dtype=torch.bfloat16)
    w = torch.zeros((128, 128), device="cuda", dtype=torch.bfloat16)
    v = torch.zeros((128,), device="cuda", dtype=torch.bfloat16)
    b = torch.zeros((8,), device="cuda")
    with pytest.raises(kvc.KvcError) as e:
        kvc.csa_compress_fused_proj_scalar(x, w, w, v, v, b, b, 1, 64, m=8)
    assert e.value.status == kvc.KVC_ERR_UNSUPPORTED
