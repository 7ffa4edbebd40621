"""GPU parity of the streaming compressor (csa_compress / hca_compress through the C ABI)
against the fp64 oracle on the same seeded inputs."""

from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from gpu_util import check_close, dev, host64, tdtype
from kv_token_compressor_b200 import kvc, synth
from oracle import compressor as O

pytestmark = pytest.mark.gpu


def _run_csa(d, m, overlap, in_dt, out_dt):
    t = {k: dev(v, in_dt) if k in ("Ca", "Cb", "Za", "Zb") else dev(v, "f32") for k, v in d.items()}
    out = kvc.csa_compress(t["Ca"], t["Cb"], t["Za"], t["Zb"], t["Ba"], t["Bb"], m=m,
                           overlap=overlap, out_dtype=tdtype(out_dt))
    torch.cuda.synchronize()
    return out


def _run_hca(d, m, in_dt, out_dt):
    out = kvc.hca_compress(dev(d["C"], in_dt), dev(d["Z"], in_dt), dev(d["B"], "f32"), m=m,
                           out_dtype=tdtype(out_dt))
    torch.cuda.synchronize()
    return out


# ------------------------------------------------------------------ the named workloads

def test_csa_f32_n1024_workload():
    w = synth.WORKLOADS["csa_f32_n1024"]
    d = synth.stream_inputs("csa", w["batch"], w["n"], w["c"], w["m"], "f32", seed=0)
    out = _run_csa(d, 4, True, "f32", "f32")
    ref = O.csa_compress(d["Ca"], d["Cb"], d["Za"], d["Zb"], d["Ba"], d["Bb"], 4, True)
    assert out.shape == (1, 256, 512)
    check_close(out, ref, "f32", "csa n=1024 fp32")


def test_hca_bf16_n65536_workload():
    w = synth.WORKLOADS["hca_bf16_n65536"]
    d = synth.stream_inputs("hca", w["batch"], w["n"], w["c"], w["m"], "bf16", seed=0)
    out = _run_hca(d, 128, "bf16", "bf16")
    ref = O.hca_compress(d["C"], d["Z"], d["B"], 128)
    assert out.shape == (1, 512, 512)
    check_close(out, ref, "bf16", "hca n=65536 bf16")


# ------------------------------------------------------------------ ragged / edge shapes

CSA_CASES = [
    # batch, n, c, m, overlap
    (3, 4 * 37 + 3, 136, 4, True),
    (2, 4 * 70, 512, 4, True),
    (1, 4 * 5, 8, 4, True),
    (2, 50, 24, 1, True),
    (2, 51, 24, 2, True),
    (2, 4 * 33 + 1, 520, 4, False),
    (2, 8 * 21 + 5, 72, 8, True),
    (1, 3 * 40 + 2, 16, 3, True),
    (2, 16 * 9, 64, 16, True),
    (2, 5 * 30 + 4, 40, 5, False),
    (1, 160 * 3, 24, 160, True),
]


@pytest.mark.parametrize("in_dt,out_dt", [("f32", "f32"), ("bf16", "bf16"), ("bf16", "f32"),
                                          ("f32", "bf16")])
@pytest.mark.parametrize("batch,n,c,m,overlap", CSA_CASES)
def test_csa_shapes(batch, n, c, m, overlap, in_dt, out_dt):
    d = synth.stream_inputs("csa", batch, n, c, m, in_dt, seed=batch * 1000 + n + c + m)
    out = _run_csa(d, m, overlap, in_dt, out_dt)
    if overlap:
        ref = O.csa_compress(d["Ca"], d["Cb"], d["Za"], d["Zb"], d["Ba"], d["Bb"], m, True)
    else:
        ref = O.csa_compress(d["Ca"], None, d["Za"], None, d["Ba"], None, m, False)
    assert out.shape == (batch, n // m, c)
    check_close(out, ref, out_dt, f"csa {batch}x{n}x{c} m={m} ov={overlap}")


HCA_CASES = [
    (2, 128 * 5 + 17, 520, 128),
    (1, 128 * 3, 8, 128),
    (3, 64 * 7 + 63, 136, 64),
    (1, 40, 24, 1),
    (2, 160 * 4, 256, 160),
    (1, 320 * 2 + 5, 16, 320),
    (1, 7 * 11, 512, 7),
    # mid-size window counts: 8 row groups per window; m = 100 leaves the row groups
    # uneven numbers of rows
    (1, 32 * 200, 256, 32),
    (1, 100 * 300 + 7, 136, 100),
]

# Window counts that make the TMA-fed window kernel pick each of its row-group splits on a
# 148-SM part (c = 512 bf16: 4 channel slabs; 148 tasks at 1, 2, 4, 8, 16 row groups per
# entry), plus a tail of n mod m rows.
TMA_RG_CASES = [
    (1, 32 * 592 + 5, 512, 32),
    (1, 32 * 296, 512, 32),
    (1, 64 * 148 + 63, 512, 64),
    (1, 128 * 74, 512, 128),
    (1, 128 * 37 + 1, 512, 128),
]


@pytest.mark.parametrize("in_dt", ["bf16", "f32"])
def test_hca_bias_not_16_byte_aligned(in_dt):
    """A bias that is 4- but not 16-byte aligned cannot be copied by the tensor engine: the
    TMA-fed window kernel then stages it with plain loads (same results)."""
    d = synth.stream_inputs("hca", 2, 128 * 300 + 9, 256, 128, in_dt, seed=31)
    Bbuf = torch.zeros(128 * 256 + 1, dtype=torch.float32, device="cuda")
    B = Bbuf[1:].view(128, 256)
    B.copy_(torch.from_numpy(d["B"]).cuda())
    assert B.data_ptr() % 16 == 4
    out = kvc.hca_compress(dev(d["C"], in_dt), dev(d["Z"], in_dt), B, m=128,
                           out_dtype=tdtype(in_dt))
    torch.cuda.synchronize()
    assert kvc.device_status() == kvc.KVC_OK
    check_close(out, O.hca_compress(d["C"], d["Z"], d["B"], 128), in_dt, "hca unaligned bias")


# CSA m = 4 problems of up to ~16 tasks (8 entries x one channel slab) per SM take the
# TMA-fed CSA kernel: several tasks per CTA, CTAs whose task range crosses a channel slab,
# entry 0 of every sequence, groups cut short by the entry count.
TMA_CSA_CASES = [
    (1, 4 * 4096 + 3, 512),
    (2, 4 * 1000 + 2, 256),
    (4, 4 * 9, 64),
]


@pytest.mark.parametrize("in_dt,out_dt", [("bf16", "bf16"), ("f32", "f32"), ("bf16", "f32")])
@pytest.mark.parametrize("batch,n,c", TMA_CSA_CASES)
def test_csa_tma_tasks(batch, n, c, in_dt, out_dt):
    d = synth.stream_inputs("csa", batch, n, c, 4, in_dt, seed=5 + n + c)
    out = _run_csa(d, 4, True, in_dt, out_dt)
    ref = O.csa_compress(d["Ca"], d["Cb"], d["Za"], d["Zb"], d["Ba"], d["Bb"], 4, True)
    assert kvc.device_status() == kvc.KVC_OK
    check_close(out, ref, out_dt, f"csa {batch}x{n}x{c}")


@pytest.mark.parametrize("in_dt,out_dt", [("bf16", "bf16"), ("f32", "f32"), ("bf16", "f32")])
@pytest.mark.parametrize("batch,n,c,m", TMA_RG_CASES)
def test_hca_row_group_splits(batch, n, c, m, in_dt, out_dt):
    d = synth.stream_inputs("hca", batch, n, c, m, in_dt, seed=11 + n + m)
    out = _run_hca(d, m, in_dt, out_dt)
    ref = O.hca_compress(d["C"], d["Z"], d["B"], m)
    assert kvc.device_status() == kvc.KVC_OK
    check_close(out, ref, out_dt, f"hca {batch}x{n}x{c} m={m}")


@pytest.mark.parametrize("in_dt,out_dt", [("f32", "f32"), ("bf16", "bf16"), ("bf16", "f32"),
                                          ("f32", "bf16")])
@pytest.mark.parametrize("batch,n,c,m", HCA_CASES)
def test_hca_shapes(batch, n, c, m, in_dt, out_dt):
    d = synth.stream_inputs("hca", batch, n, c, m, in_dt, seed=7 + n + c + m)
    out = _run_hca(d, m, in_dt, out_dt)
    ref = O.hca_compress(d["C"], d["Z"], d["B"], m)
    assert out.shape == (batch, n // m, c)
    check_close(out, ref, out_dt, f"hca {batch}x{n}x{c} m={m}")


@pytest.mark.parametrize("profile", ["ramp", "late_jump", "falling", "ramp_below_headroom"])
def test_hca_reference_moves(profile):
    """The TMA-fed window kernel moves its softmax reference only when a chunk's logit bound
    exceeds it by more than its headroom: logits that climb across a window (by ~2 log2
    units a row, or just under the headroom per 8-row chunk), one very large late row, and
    logits that fall (later chunks far below the reference) all pool like the fp64 oracle."""
    m, c = 128, 256
    h = synth.stream_inputs("hca", 2, m * 40 + 3, c, m, "f32", seed=41)
    rows = np.arange(h["Z"].shape[1]) % m
    ln2 = np.log(2.0)
    if profile == "ramp":
        shift = 2.0 * rows * ln2                   # +2 log2 units per row
    elif profile == "late_jump":
        shift = np.where(rows == m - 1, 100.0, 0.0)  # one row ~144 log2 units up
    elif profile == "falling":
        shift = -1.5 * rows                        # later chunks far below the first
    else:
        shift = 15.5 * ln2 * (rows // 8) / 1.0     # each chunk just under 16 log2 units up
    h["Z"] = (h["Z"] + shift[None, :, None]).astype(np.float32)
    out = _run_hca(h, m, "f32", "f32")
    assert kvc.device_status() == kvc.KVC_OK
    check_close(out, O.hca_compress(h["C"], h["Z"], h["B"], m), "f32", f"hca reference {profile}")


def test_wide_logit_range():
    """Row offsets of +-30 on the logits: the max subtraction must keep exp2 finite."""
    d = synth.stream_inputs("csa", 2, 4 * 64, 64, 4, "f32", seed=3, z_row_offset=30.0)
    out = _run_csa(d, 4, True, "f32", "f32")
    ref = O.csa_compress(d["Ca"], d["Cb"], d["Za"], d["Zb"], d["Ba"], d["Bb"], 4, True)
    check_close(out, ref, "f32", "csa wide logits")
    h = synth.stream_inputs("hca", 1, 512, 64, 128, "f32", seed=4, z_row_offset=30.0)
    out = _run_hca(h, 128, "f32", "f32")
    check_close(out, O.hca_compress(h["C"], h["Z"], h["B"], 128), "f32", "hca wide logits")


@pytest.mark.parametrize("spread", [38.0, 90.0])
@pytest.mark.parametrize("mode,batch,n,c,m", [
    ("hca", 1, 128 * 6 + 5, 136, 128),   # few windows: row groups merged in shared memory
    ("hca", 1, 16 * 15000, 64, 16),       # many windows: one per thread, several chunks
    ("csa", 2, 8 * 40 + 3, 72, 8),        # two segments (a then b) in the window kernel
])
def test_bias_spread_paths(mode, batch, n, c, m, spread):
    """Biases uniform in [-spread/2, spread/2] (natural-log units).  38 stays inside the
    spread (64 in log2 units) where the window kernel bounds each chunk's maximum by
    max(z) + max(b); 90 is beyond it and takes the exact per-row maximum.  Both must
    match the oracle, although the bounded maximum leaves weights as small as 2^-55."""
    rng = np.random.default_rng(int(spread) + m)
    d = synth.stream_inputs(mode, batch, n, c, m, "f32", seed=int(spread) + n)
    for k in [k for k in d if k.startswith("B")]:
        d[k] = rng.uniform(-spread / 2, spread / 2, size=d[k].shape).astype(np.float32)
    if mode == "hca":
        out = _run_hca(d, m, "f32", "f32")
        ref = O.hca_compress(d["C"], d["Z"], d["B"], m)
    else:
        out = _run_csa(d, m, True, "f32", "f32")
        ref = O.csa_compress(d["Ca"], d["Cb"], d["Za"], d["Zb"], d["Ba"], d["Bb"], m, True)
    check_close(out, ref, "f32", f"{mode} m={m} bias spread {spread}")


@pytest.mark.parametrize("seed", range(6))
def test_random_shapes_across_dispatch(seed):
    """Seeded random problems across the dispatch boundaries: CSA with m in {1, 2, 4, 8, 13}
    (with and without overlap) and HCA with m in {8, 16, 32, 64, 128, 150}; c any multiple
    of 8 up to 1024, ragged n, 1-3 sequences, every input/output dtype pair.  Each output
    lies between canary bands that must come back untouched."""
    rng = np.random.default_rng(500 + seed)
    for _ in range(4):
        batch = int(rng.integers(1, 4))
        c = 8 * int(rng.integers(1, 129))
        in_dt, out_dt = rng.choice(["bf16", "f32"]), rng.choice(["bf16", "f32"])
        if rng.random() < 0.5:
            m = int(rng.choice([1, 2, 4, 8, 13]))
            overlap = bool(rng.random() < 0.7)
            n = int(rng.integers(m, min(6000, 2_000_000 // c)))
            d = synth.stream_inputs("csa", batch, n, c, m, in_dt, seed=seed * 17 + m)
            t = {k: dev(v, in_dt) if k in ("Ca", "Cb", "Za", "Zb") else dev(v, "f32")
                 for k, v in d.items()}
            ne = n // m
            buf = torch.full((batch * ne * c + 128,), -777.0, device="cuda", dtype=tdtype(out_dt))
            out = buf[64:64 + batch * ne * c].view(batch, ne, c)
            kvc.csa_compress(t["Ca"], t["Cb"], t["Za"], t["Zb"], t["Ba"], t["Bb"], m=m,
                             overlap=overlap, out=out, out_dtype=tdtype(out_dt))
            ref = O.csa_compress(d["Ca"], d["Cb"], d["Za"], d["Zb"], d["Ba"], d["Bb"], m, overlap)
            what = f"csa b={batch} n={n} c={c} m={m} ov={overlap} {in_dt}->{out_dt} ({kvc.last_kernel()})"
        else:
            m = int(rng.choice([8, 16, 32, 64, 128, 150]))
            n = int(rng.integers(m, min(40 * m, 4_000_000 // c)))
            d = synth.stream_inputs("hca", batch, n, c, m, in_dt, seed=seed * 19 + m)
            ne = n // m
            buf = torch.full((batch * ne * c + 128,), -777.0, device="cuda", dtype=tdtype(out_dt))
            out = buf[64:64 + batch * ne * c].view(batch, ne, c)
            kvc.hca_compress(dev(d["C"], in_dt), dev(d["Z"], in_dt), dev(d["B"], "f32"), m=m, out=out,
                             out_dtype=tdtype(out_dt))
            ref = O.hca_compress(d["C"], d["Z"], d["B"], m)
            what = f"hca b={batch} n={n} c={c} m={m} {in_dt}->{out_dt} ({kvc.last_kernel()})"
        assert kvc.device_status() == kvc.KVC_OK, what
        check_close(out, ref, out_dt, what)
        assert bool(torch.all(buf[:64] == -777.0)) and bool(torch.all(buf[64 + batch * ne * c:] == -777.0)), what


def test_boundary_and_mean_on_gpu():
    """Closed forms on the kernel itself: entry 0 ignores the b-streams; constant logits
    with zero bias give the mean of the window (1/8 and 1/4 weights are exact)."""
    d = synth.stream_inputs("csa", 1, 64, 32, 4, "f32", seed=5)
    d["Za"][:] = 0.25
    d["Zb"][:] = 0.25
    d["Ba"][:] = 0
    d["Bb"][:] = 0
    out = host64(_run_csa(d, 4, True, "f32", "f32"))[0]
    assert np.allclose(out[0], d["Ca"][0, :4].astype(np.float64).mean(0), rtol=0, atol=2e-6)
    for i in (1, 7, 15):
        w = np.vstack([d["Ca"][0, 4 * i:4 * i + 4], d["Cb"][0, 4 * i - 4:4 * i]]).astype(np.float64)
        assert np.allclose(out[i], w.mean(0), rtol=0, atol=2e-6)
    d2 = {k: v.copy() for k, v in d.items()}
    d2["Cb"][:] = 1e6
    out2 = host64(_run_csa(d2, 4, True, "f32", "f32"))[0]
    assert np.array_equal(out2[0], out[0])


def test_empty_problem_returns_empty():
    x = torch.zeros((2, 3, 64), device="cuda", dtype=torch.bfloat16)
    b = torch.zeros((4, 64), device="cuda")
    out = kvc.csa_compress(x, x, x, x, b, b, m=4)
    assert out.shape == (2, 0, 64)
    out = kvc.hca_compress(x, x, torch.zeros((128, 64), device="cuda"), m=128)
    assert out.shape == (2, 0, 64)


def test_host_pointer_is_rejected():
    """A host buffer handed to the ABI is refused on the host, never dereferenced."""
    L = kvc.lib()
    host = torch.zeros((1, 64, 64), dtype=torch.float32).pin_memory()
    dv = torch.zeros((1, 64, 64), device="cuda")
    b = torch.zeros((4, 64), device="cuda")
    out = torch.empty((1, 16, 64), device="cuda")
    plain = np.zeros(64 * 64 + 16, np.float32)
    hp = plain.ctypes.data + (-plain.ctypes.data) % 16
    for bad in (hp,):
        st = L.csa_compress(bad, dv.data_ptr(), dv.data_ptr(), dv.data_ptr(), kvc.KVC_F32,
                            b.data_ptr(), b.data_ptr(), 1, 64, 64, 4, 1, out.data_ptr(), kvc.KVC_F32,
                            None)
        assert st == kvc.KVC_ERR_POINTER
    st = L.hca_compress(dv.data_ptr(), dv.data_ptr(), kvc.KVC_F32, b.data_ptr(), 1, 64, 64, 4,
                        host.data_ptr(), kvc.KVC_F32, None)
    assert st == kvc.KVC_ERR_POINTER
    assert kvc.device_status() == kvc.KVC_OK


# ------------------------------------------------------------------ full size, every entry

CHUNK = 1 << 14  # entries per host comparison (65536 tokens of CSA)


def _host_rows(t, lo, hi):
    return t[0, lo:hi].float().cpu().numpy()[None]


@pytest.fixture(scope="module")
def long_inputs():
    w = synth.WORKLOADS["csa_long_n1048576"]
    t = synth.stream_inputs_torch("csa", 1, w["n"], w["c"], 4, "bf16", seed=0,
                                  z_row_offset=w["z_row_offset"])
    g = torch.Generator(device="cuda")
    g.manual_seed(1)
    t["B_hca"] = torch.randn((128, w["c"]), generator=g, device="cuda") * float(np.sqrt(0.1))
    yield t
    del t
    torch.cuda.empty_cache()


def test_csa_long_n1048576_every_entry(long_inputs):
    """The long-context workload (n = 2^20, c = 512, bf16 streams with per-row logit
    offsets), CSA m = 4: all 262,144 entries against the oracle, in chunks of 16,384
    entries whose host copy starts one block early (the b-rows of the chunk's first
    entry)."""
    t = long_inputs
    out = kvc.csa_compress(t["Ca"], t["Cb"], t["Za"], t["Zb"], t["Ba"], t["Bb"], m=4,
                           out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    ne = (1 << 20) // 4
    assert out.shape == (1, ne, 512)
    Ba, Bb = host64(t["Ba"]), host64(t["Bb"])
    for i0 in range(0, ne, CHUNK):
        i1 = min(ne, i0 + CHUNK)
        lo = 4 * (i0 - 1) if i0 > 0 else 0
        mini = {k: _host_rows(t[k], lo, 4 * i1) for k in ("Ca", "Cb", "Za", "Zb")}
        j0 = 1 if i0 > 0 else 0  # entry i0 is entry j0 of the chunk's rows
        ref = O.csa_compress(mini["Ca"], mini["Cb"], mini["Za"], mini["Zb"], Ba, Bb, 4, True,
                             entries=[(0, j0 + k) for k in range(i1 - i0)])
        check_close(out[0, i0:i1], ref, "bf16", f"csa n=2^20 entries {i0}..{i1 - 1}")


def test_hca_long_n1048576_every_entry(long_inputs):
    """HCA m' = 128 on the same streams (C := C^a, Z := Z^a, its own bias): all 8,192
    entries against the oracle."""
    t = long_inputs
    out = kvc.hca_compress(t["Ca"], t["Za"], t["B_hca"], m=128, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    ne = (1 << 20) // 128
    assert out.shape == (1, ne, 512)
    B = host64(t["B_hca"])
    step = CHUNK // 16  # 1024 entries = 131072 rows per chunk
    for i0 in range(0, ne, step):
        i1 = min(ne, i0 + step)
        C = _host_rows(t["Ca"], 128 * i0, 128 * i1)
        Z = _host_rows(t["Za"], 128 * i0, 128 * i1)
        check_close(out[0, i0:i1], O.hca_compress(C, Z, B, 128)[0], "bf16",
                    f"hca n=2^20 entries {i0}..{i1 - 1}")


def test_long_weights_sum_to_one(long_inputs):
    """Property at full size: with every value row equal to 1 the output is 1 everywhere
    (weights of each (entry, channel) sum to one, entry 0 included)."""
    t = long_inputs
    ones = torch.ones_like(t["Ca"])
    out = kvc.csa_compress(ones, ones, t["Za"], t["Zb"], t["Ba"], t["Bb"], m=4,
                           out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.max(torch.abs(out - 1.0)).item() < 2e-6
    out = kvc.hca_compress(ones, t["Za"], t["B_hca"], m=128, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.max(torch.abs(out - 1.0)).item() < 2e-6


def test_shard_plan_on_gpu_is_bit_exact():
    """Each rank's planned rows (one-block halo included), compressed on their own with
    the halo entry dropped, give exactly the full run's entries."""
    from kv_token_compressor_b200 import shard

    n, c = 4 * 1000 + 3, 512
    d = synth.stream_inputs("csa", 1, n, c, 4, "bf16", seed=21)
    t = {k: dev(v, "bf16") if v.ndim == 3 else dev(v, "f32") for k, v in d.items()}
    full = kvc.csa_compress(t["Ca"], t["Cb"], t["Za"], t["Zb"], t["Ba"], t["Bb"], m=4)
    parts = []
    for s in shard.plan(n, 4, 3, True):
        loc = {k: (v[:, s.row0:s.row1].contiguous() if v.dim() == 3 else v) for k, v in t.items()}
        o = kvc.csa_compress(loc["Ca"], loc["Cb"], loc["Za"], loc["Zb"], loc["Ba"], loc["Bb"], m=4)
        parts.append(o[:, 1:] if s.drop_first else o)
    torch.cuda.synchronize()
    assert torch.equal(torch.cat(parts, dim=1), full)
