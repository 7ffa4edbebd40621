"""GPU parity of the entry-list calls (csa_compress_entries / hca_compress_entries):
ragged prefill, decode-style lists, agreement with the dense calls (to bf16 rounding: the
dense calls may take other kernels with another summation order), and out-of-range entries
that the kernel skips and reports."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from gpu_util import check_close, dev, tdtype
from kv_token_compressor_b200 import kvc, synth
from oracle import compressor as O

pytestmark = pytest.mark.gpu


def _pack(lens, c, m, dt, seed, mode="csa"):
    d = synth.stream_inputs(mode, 1, int(sum(lens)), c, m, dt, seed=seed)
    starts = np.concatenate([[0], np.cumsum(lens)[:-1]]).astype(np.int64)
    return d, starts


def _list(starts, lens, ents):
    seq_start = torch.tensor([starts[s] for s, _ in ents], dtype=torch.int64, device="cuda")
    seq_len = torch.tensor([lens[s] for s, _ in ents], dtype=torch.int64, device="cuda")
    entry = torch.tensor([e for _, e in ents], dtype=torch.int64, device="cuda")
    return seq_start, seq_len, entry


def _csa_ref(d, starts, lens, ents, m):
    rows = []
    for s, e in ents:
        sl = slice(starts[s], starts[s] + lens[s])
        rows.append(O.csa_compress(d["Ca"][:, sl], d["Cb"][:, sl], d["Za"][:, sl], d["Zb"][:, sl],
                                   d["Ba"], d["Bb"], m, True, entries=[(0, e)])[0])
    return np.array(rows)


@pytest.mark.parametrize("m,dt", [(4, "bf16"), (4, "f32"), (2, "bf16"), (8, "bf16")])
def test_ragged_prefill(m, dt):
    lens = [m * 37 + 3, m * 5, m * 100, m - 1, m * 2]
    c = 136
    d, starts = _pack(lens, c, m, dt, seed=1)
    ents = [(s, e) for s, L in enumerate(lens) for e in range(L // m)]
    t = {k: dev(v[0], dt) if v.ndim == 3 else dev(v, "f32") for k, v in d.items()}
    lst = _list(starts, lens, ents)
    out = kvc.csa_compress_entries(t["Ca"], t["Cb"], t["Za"], t["Zb"], t["Ba"], t["Bb"], *lst, m=m,
                                   out_dtype=tdtype(dt))
    assert kvc.device_status() == kvc.KVC_OK
    check_close(out, _csa_ref(d, starts, lens, ents, m), dt, f"ragged m={m}")


def test_decode_lists_last_entries():
    """Decode: sequences of different lengths; each lists only its newest complete entry
    (the entry whose a-block just filled), in a shuffled order."""
    m, c = 4, 512
    rng = np.random.default_rng(2)
    lens = [int(x) for x in rng.integers(4, 4000, size=37)]
    d, starts = _pack(lens, c, m, "bf16", seed=2)
    ents = [(s, L // m - 1) for s, L in enumerate(lens)]
    rng.shuffle(ents)
    t = {k: dev(v[0], "bf16") if v.ndim == 3 else dev(v, "f32") for k, v in d.items()}
    out = kvc.csa_compress_entries(t["Ca"], t["Cb"], t["Za"], t["Zb"], t["Ba"], t["Bb"],
                                   *_list(starts, lens, ents), m=4)
    assert kvc.device_status() == kvc.KVC_OK
    check_close(out, _csa_ref(d, starts, lens, ents, m), "bf16", "decode lists")


def test_lists_equal_dense_calls():
    batch, n, c = 3, 4 * 300 + 1, 512
    d = synth.stream_inputs("csa", batch, n, c, 4, "bf16", seed=3)
    t = {k: dev(v, "bf16") if v.ndim == 3 else dev(v, "f32") for k, v in d.items()}
    dense = kvc.csa_compress(t["Ca"], t["Cb"], t["Za"], t["Zb"], t["Ba"], t["Bb"], m=4)
    flat = {k: t[k].reshape(batch * n, c) for k in ("Ca", "Cb", "Za", "Zb")}
    ne = n // 4
    ents = [(b, i) for b in range(batch) for i in range(ne)]
    starts, lens = [b * n for b in range(batch)], [n] * batch
    out = kvc.csa_compress_entries(flat["Ca"], flat["Cb"], flat["Za"], flat["Zb"], t["Ba"], t["Bb"],
                                   *_list(starts, lens, ents), m=4)
    torch.cuda.synchronize()
    # the dense call runs the TMA-fed kernel, which adds the a- and b-block sums of a window
    # in another order than the listed kernel: equal to bf16 rounding, not bit for bit
    diff = (out.reshape(batch, ne, c).float() - dense.float()).abs()
    assert torch.all(diff <= 2.0 ** -7 * dense.float().abs() + 1e-6).item()
    # HCA
    h = synth.stream_inputs("hca", batch, 128 * 9 + 5, c, 128, "bf16", seed=4)
    th = {k: dev(v, "bf16") if v.ndim == 3 else dev(v, "f32") for k, v in h.items()}
    dense = kvc.hca_compress(th["C"], th["Z"], th["B"], m=128)
    nh = 128 * 9 + 5
    ents = [(b, i) for b in range(batch) for i in range(9)]
    out = kvc.hca_compress_entries(th["C"].reshape(-1, c), th["Z"].reshape(-1, c), th["B"],
                                   *_list([b * nh for b in range(batch)], [nh] * batch, ents), m=128)
    torch.cuda.synchronize()
    # the dense call splits these few windows over row groups (a different summation
    # order), so the two agree to bf16 rounding rather than bit for bit
    diff = (out.reshape(batch, 9, c).float() - dense.float()).abs()
    assert torch.all(diff <= 2.0 ** -7 * dense.float().abs() + 1e-6).item()


def test_out_of_range_entries_are_skipped_and_reported():
    m, c = 4, 64
    lens = [40, 24]
    d, starts = _pack(lens, c, m, "f32", seed=5)
    t = {k: dev(v[0], "f32") if v.ndim == 3 else dev(v, "f32") for k, v in d.items()}
    total = sum(lens)
    good = [(0, 3), (1, 5), (0, 0)]
    rows = [(starts[s], lens[s], e) for s, e in good]
    bad = [(0, 40, 10),          # entry 10 needs rows up to 43 > length 40
           (30, 40, 0),          # sequence runs past the streams (30 + 40 > 64)
           (-4, 8, 0),           # negative start
           (0, 40, -1)]          # negative entry
    allr = rows[:1] + bad[:2] + rows[1:] + bad[2:]
    seq_start = torch.tensor([r[0] for r in allr], dtype=torch.int64, device="cuda")
    seq_len = torch.tensor([r[1] for r in allr], dtype=torch.int64, device="cuda")
    entry = torch.tensor([r[2] for r in allr], dtype=torch.int64, device="cuda")
    out = torch.full((len(allr), c), 12345.0, device="cuda")
    kvc.csa_compress_entries(t["Ca"], t["Cb"], t["Za"], t["Zb"], t["Ba"], t["Bb"], seq_start, seq_len,
                             entry, m=4, out=out, out_dtype=torch.float32)
    assert kvc.device_status() == kvc.KVC_ERR_INDEX
    assert kvc.device_status() == kvc.KVC_OK  # the report clears the word
    got = out.cpu().numpy()
    ref = _csa_ref(d, starts, lens, good, m)
    check_close(torch.from_numpy(got[[0, 3, 4]]), ref, "f32", "valid rows among bad ones")
    assert np.all(got[[1, 2, 5, 6]] == 12345.0)
    # HCA lists are checked the same way
    h = synth.stream_inputs("hca", 1, 256, c, 128, "f32", seed=6)
    th = {k: dev(v[0], "f32") if v.ndim == 3 else dev(v, "f32") for k, v in h.items()}
    s0 = torch.tensor([0, 0], dtype=torch.int64, device="cuda")
    ln = torch.tensor([256, 256], dtype=torch.int64, device="cuda")
    en = torch.tensor([1, 2], dtype=torch.int64, device="cuda")
    kvc.hca_compress_entries(th["C"], th["Z"], th["B"], s0, ln, en, m=128)
    assert kvc.device_status() == kvc.KVC_ERR_INDEX


@pytest.mark.parametrize("seed", range(4))
def test_random_lists(seed):
    """Seeded random entry lists over ragged packed sequences: CSA with m in {2, 4, 8}
    (with and without overlap) and HCA with m in {16, 64, 128}; random entries of every
    sequence, entry 0 included, in a shuffled order; every input/output dtype pair."""
    rng = np.random.default_rng(700 + seed)
    for mode in ("csa", "hca"):
        m = int(rng.choice([2, 4, 8] if mode == "csa" else [16, 64, 128]))
        c = 8 * int(rng.integers(1, 97))
        in_dt, out_dt = rng.choice(["bf16", "f32"]), rng.choice(["bf16", "f32"])
        lens = [int(x) for x in rng.integers(m, 30 * m, size=int(rng.integers(1, 9)))]
        d, starts = _pack(lens, c, m, in_dt, seed=seed * 13 + m, mode=mode)
        ents = [(s, int(e)) for s, L in enumerate(lens)
                for e in rng.choice(L // m, size=min(L // m, 5), replace=False)]
        ents.append((0, 0))
        rng.shuffle(ents)
        lst = _list(starts, lens, ents)
        if mode == "csa":
            overlap = bool(rng.random() < 0.7)
            t = {k: dev(v[0], in_dt) if v.ndim == 3 else dev(v, "f32") for k, v in d.items()}
            out = kvc.csa_compress_entries(t["Ca"], t["Cb"], t["Za"], t["Zb"], t["Ba"], t["Bb"], *lst,
                                           m=m, overlap=overlap, out_dtype=tdtype(out_dt))
            ref = []
            for s_, e in ents:
                sl = slice(starts[s_], starts[s_] + lens[s_])
                ref.append(O.csa_compress(d["Ca"][:, sl], d["Cb"][:, sl], d["Za"][:, sl], d["Zb"][:, sl],
                                          d["Ba"], d["Bb"], m, overlap, entries=[(0, e)])[0])
        else:
            t = {k: dev(v[0], in_dt) if v.ndim == 3 else dev(v, "f32") for k, v in d.items()}
            out = kvc.hca_compress_entries(t["C"], t["Z"], t["B"], *lst, m=m, out_dtype=tdtype(out_dt))
            ref = []
            for s_, e in ents:
                sl = slice(starts[s_], starts[s_] + lens[s_])
                ref.append(O.hca_compress(d["C"][:, sl], d["Z"][:, sl], d["B"], m)[0, e])
        what = f"{mode} lists m={m} c={c} {in_dt}->{out_dt} ({kvc.last_kernel()})"
        assert kvc.device_status() == kvc.KVC_OK, what
        check_close(out, np.array(ref), out_dt, what)


def test_sync_check_reports_from_the_call():
    """With the sync check on, the call that named an out-of-range entry raises
    KVC_ERR_INDEX itself (and clears the word); a valid call passes."""
    m, c = 4, 64
    lens = [40, 12]
    d, starts = _pack(lens, c, m, "f32", seed=11)
    t = {k: dev(v[0], "f32") if v.ndim == 3 else dev(v, "f32") for k, v in d.items()}
    args = (t["Ca"], t["Cb"], t["Za"], t["Zb"], t["Ba"], t["Bb"])
    kvc.set_sync_check(True)
    try:
        with pytest.raises(kvc.KvcError) as e:
            kvc.csa_compress_entries(*args, *_list(starts, lens, [(0, 3), (1, 5)]), m=4)
        assert e.value.status == kvc.KVC_ERR_INDEX
        assert kvc.device_status() == kvc.KVC_OK
        ents = [(0, 3), (1, 2)]
        out = kvc.csa_compress_entries(*args, *_list(starts, lens, ents), m=4,
                                       out_dtype=torch.float32)
        check_close(out, _csa_ref(d, starts, lens, ents, m), "f32", "sync-checked call")
    finally:
        kvc.set_sync_check(False)
    assert not kvc.sync_check()


def test_empty_list():
    x = torch.zeros((16, 64), device="cuda")
    b = torch.zeros((4, 64), device="cuda")
    e = torch.zeros((0,), dtype=torch.int64, device="cuda")
    out = kvc.csa_compress_entries(x, x, x, x, b, b, e, e, e, m=4)
    assert out.shape == (0, 64)
