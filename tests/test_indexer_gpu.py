"""GPU parity of the lightning indexer (lightning_indexer_scores / indexer_topk through the C
ABI) against the fp64 oracle on the same seeded inputs.

Scores are fp32 outputs: within 1e-5 of the row's largest |score| of the oracle.  The
top-k is compared bit for bit with the oracle's selection over the SAME fp32 scores the
kernel was given (several entries can share a score; the order is fixed by the index), and
end to end against the oracle's fp64 scores up to the scores' own rounding."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from kv_token_compressor_b200 import kvc, synth
from oracle import indexer as IX

pytestmark = pytest.mark.gpu


def _dev(d):
    return {"q": torch.from_numpy(d["q"]).cuda().to(torch.bfloat16),
            "K": torch.from_numpy(d["K"]).cuda().to(torch.bfloat16),
            "w": torch.from_numpy(d["w"]).cuda()}


def _i64(xs):
    return torch.tensor(list(xs), dtype=torch.int64, device="cuda")


def _scores(t, ks, nv, max_visible, ld=None, fill=-12345.0):
    T = t["q"].shape[0]
    ld = ld or max(4, -(-max_visible // 4) * 4)
    out = torch.full((T, ld), fill, dtype=torch.float32, device="cuda")
    kvc.lightning_indexer_scores(t["q"], t["w"], t["K"], _i64(ks), _i64(nv), max_visible, scores=out)
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("H", [64, 16, 48, 128])
def test_scores_windows(H):
    rows = 3000
    d = synth.indexer_inputs(5, H, rows, seed=H)
    t = _dev(d)
    ks = [0, 100, 2999, 1500, 7]
    nv = [3000, 1029, 1, 0, 128]
    out = _scores(t, ks, nv, 3000)
    assert kvc.device_status() == kvc.KVC_OK
    ref = IX.indexer_scores(d["q"], d["w"], d["K"], ks, nv)
    got = out.cpu().numpy()
    for i in range(5):
        r = ref[i]
        if len(r):
            tol = 1e-5 * max(np.max(np.abs(r)), 1e-30)
            assert np.max(np.abs(got[i, :nv[i]] - r)) <= tol, (H, i)
        assert np.all(got[i, nv[i]:3000] == -12345.0), "entries past n_visible were written"


def test_scores_bad_window_is_skipped_and_reported():
    d = synth.indexer_inputs(3, 64, 500, seed=1)
    t = _dev(d)
    ks, nv = [0, 450, 10], [300, 100, 20]  # query 1 runs past the keys
    out = _scores(t, ks, nv, 300)
    assert kvc.device_status() == kvc.KVC_ERR_INDEX
    assert kvc.device_status() == kvc.KVC_OK
    got = out.cpu().numpy()
    assert np.all(got[1] == -12345.0)
    ref = IX.indexer_scores(d["q"][[0, 2]], d["w"][[0, 2]], d["K"], [0, 10], [300, 20])
    assert np.allclose(got[0, :300], ref[0], rtol=0, atol=1e-5 * np.max(np.abs(ref[0])))
    assert np.allclose(got[2, :20], ref[1], rtol=0, atol=1e-5 * np.max(np.abs(ref[1])))
    # n_visible above max_visible is refused the same way
    out2 = torch.full((1, 300), -1.0, device="cuda")
    tt = {k: v[:1] for k, v in t.items() if k != "K"}
    kvc.lightning_indexer_scores(tt["q"], tt["w"], t["K"], _i64([0]), _i64([300]), 200, scores=out2)
    assert kvc.device_status() == kvc.KVC_ERR_INDEX
    assert torch.all(out2 == -1.0).item()


def _topk_gpu(scores, nv, k, max_visible):
    idx, val = kvc.indexer_topk(scores, _i64(nv), k, max_visible)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), val.cpu().numpy()


@pytest.mark.parametrize("k", [1, 7, 512, 1024, 2048])
@pytest.mark.parametrize("kind", ["ties", "continuous", "sorted"])
def test_topk_exact_given_scores(k, kind):
    rng = np.random.default_rng(k + len(kind))
    nv = [0, 1, 5, 1000, 4099, 100003, 327680]
    ld = 327680
    S = np.full((len(nv), ld), np.nan, dtype=np.float32)  # past n_visible: never read
    for i, n in enumerate(nv):
        if kind == "ties":  # few distinct values, many exact zeros (as ReLU makes)
            v = rng.integers(-2, 5, size=n).astype(np.float32)
            v[rng.random(n) < 0.5] = 0.0
        else:
            v = rng.standard_normal(n).astype(np.float32)
        if kind == "sorted":  # the largest scores crowd into the last warps of the last CTA
            v = np.sort(v)
        S[i, :n] = v
    idx, val = _topk_gpu(torch.from_numpy(S).cuda(), nv, k, ld)
    assert kvc.device_status() == kvc.KVC_OK
    for i, n in enumerate(nv):
        ref_idx, ref_val = IX.topk_row(S[i, :n].astype(np.float64), k)
        assert np.array_equal(idx[i], ref_idx), (k, kind, n)
        assert np.array_equal(val[i].astype(np.float64), ref_val), (k, kind, n)


def test_topk_many_rows_in_waves():
    """More rows than clusters resident at once (the launch runs in waves); each row its own
    length and distribution."""
    rng = np.random.default_rng(40)
    T, ld, k = 40, 65536, 1024
    nv = [int(x) for x in rng.integers(0, ld + 1, size=T)]
    nv[0], nv[1] = ld, 0
    S = np.zeros((T, ld), dtype=np.float32)
    for i, n in enumerate(nv):
        S[i, :n] = rng.standard_normal(n) * (1 + i % 5) + (i % 3)
    idx, val = _topk_gpu(torch.from_numpy(S).cuda(), nv, k, ld)
    assert kvc.device_status() == kvc.KVC_OK
    for i, n in enumerate(nv):
        ref_idx, ref_val = IX.topk_row(S[i, :n].astype(np.float64), k)
        assert np.array_equal(idx[i], ref_idx), (i, n)
        assert np.array_equal(val[i].astype(np.float64), ref_val), (i, n)


@pytest.mark.parametrize("k", [1, 1024, 2048])
def test_topk_all_scores_equal(k):
    """Every score the same: the selection is the first k indices in order (every warp's
    candidate list overflows; the rank has one bin)."""
    nv = [327680, 4099, 2048]
    S = np.full((len(nv), 327680), 2.5, dtype=np.float32)
    idx, val = _topk_gpu(torch.from_numpy(S).cuda(), nv, k, 327680)
    assert kvc.device_status() == kvc.KVC_OK
    for i, n in enumerate(nv):
        want = np.arange(k) if k <= n else np.concatenate([np.arange(n), -np.ones(k - n)])
        assert np.array_equal(idx[i], want.astype(np.int32)), (k, n)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_topk_randomized_rows(seed):
    """Seeded random batches: per row a length in [0, 327680], a distribution (continuous,
    few values with many zeros, ascending runs, constant blocks with noise) and one k per
    launch in [1, 2048]; every row bit for bit against the oracle's selection."""
    rng = np.random.default_rng(1000 + seed)
    T, ld = 16, 327680
    k = int(rng.integers(1, 2049))
    nv = [int(x) for x in rng.integers(0, ld + 1, size=T)]
    nv[int(rng.integers(T))] = ld
    S = np.full((T, ld), np.nan, dtype=np.float32)
    for i, n in enumerate(nv):
        kind = i % 4
        if kind == 0:
            v = rng.standard_normal(n) * rng.uniform(0.01, 100)
        elif kind == 1:
            v = rng.integers(-3, 4, size=n).astype(np.float64)
            v[rng.random(n) < 0.6] = 0.0
        elif kind == 2:
            v = np.cumsum(rng.random(n)) * rng.choice([-1, 1])
        else:
            v = np.repeat(rng.standard_normal(max(1, n // 1000 + 1)), 1000)[:n]
            v = v + (rng.random(n) < 0.01) * rng.standard_normal(n)
        S[i, :n] = v.astype(np.float32)
    idx, val = _topk_gpu(torch.from_numpy(S).cuda(), nv, k, ld)
    assert kvc.device_status() == kvc.KVC_OK
    for i, n in enumerate(nv):
        ref_idx, ref_val = IX.topk_row(S[i, :n].astype(np.float64), k)
        assert np.array_equal(idx[i], ref_idx), (seed, i, n, k)
        assert np.array_equal(val[i].astype(np.float64), ref_val), (seed, i, n, k)


def test_topk_signed_zero_and_negatives():
    """-0.0 and 0.0 are the same score (ties by index); negative scores order correctly."""
    v = np.array([0.0, -0.0, -1.5, 2.0, -0.0, 0.0, -3.0, 2.0, -1.5], dtype=np.float32)
    S = np.zeros((1, 12), dtype=np.float32)
    S[0, :9] = v
    idx, val = _topk_gpu(torch.from_numpy(S).cuda(), [9], 7, 9)
    assert idx[0].tolist() == [3, 7, 0, 1, 4, 5, 2]
    assert val[0].tolist()[:2] == [2.0, 2.0]


def test_topk_row_past_max_visible_is_reported():
    S = torch.zeros((2, 8), device="cuda")
    idx = torch.full((2, 4), 77, dtype=torch.int32, device="cuda")
    kvc.indexer_topk(S, _i64([8, 3]), 4, 4, out_idx=idx)
    assert kvc.device_status() == kvc.KVC_ERR_INDEX
    assert idx[0].tolist() == [77] * 4          # skipped row untouched
    assert idx[1].tolist() == [0, 1, 2, -1]


def test_scores_then_topk_on_a_user_stream():
    """The top-k launches as a programmatic dependent of the kernel ahead of it: on a
    stream of the caller's, back to back with the score kernel and with new inputs each
    time, it must select from the scores just written (compared bit for bit with the
    oracle's selection over those scores)."""
    T, H, S, k = 3, 64, 1 << 16, 512
    s = torch.cuda.Stream()
    ks, nv = [i * S for i in range(T)], [S, S - 7, 40000]
    out = torch.empty((T, S), dtype=torch.float32, device="cuda")
    with torch.cuda.stream(s):
        for it in range(4):
            t = synth.indexer_inputs_torch(T, H, T * S, seed=50 + it)
            kvc.lightning_indexer_scores(t["q"], t["w"], t["K"], _i64(ks), _i64(nv), S, scores=out)
            idx, _ = kvc.indexer_topk(out, _i64(nv), k, S)
            s.synchronize()
            got, gidx = out.cpu().numpy(), idx.cpu().numpy()
            for i in range(T):
                ref_idx, _ = IX.topk_row(got[i, :nv[i]].astype(np.float64), k)
                assert np.array_equal(gidx[i], ref_idx), (it, i)
    assert kvc.device_status(s) == kvc.KVC_OK


def test_decode_step_end_to_end():
    """A decode step: 4 sequences of 2^20 tokens (262144 compressed keys each), one query
    of 64 heads per sequence, k = 1024.  Full score rows against the fp64 oracle, the top-k
    bit-exact on the kernel's scores, and against the oracle's fp64 scores up to rounding."""
    T, H, S, k = 4, 64, 262144, 1024
    t = synth.indexer_inputs_torch(T, H, T * S, seed=5)
    ks, nv = [i * S for i in range(T)], [S, S - 1, S - 1000, 77777]
    out = torch.empty((T, S), dtype=torch.float32, device="cuda")
    kvc.lightning_indexer_scores(t["q"], t["w"], t["K"], _i64(ks), _i64(nv), S, scores=out)
    idx, val = kvc.indexer_topk(out, _i64(nv), k, S)
    torch.cuda.synchronize()
    assert kvc.device_status() == kvc.KVC_OK
    q = t["q"].float().cpu().numpy()
    w = t["w"].cpu().numpy()
    K = t["K"].float().cpu().numpy()
    got = out.cpu().numpy()
    gidx = idx.cpu().numpy()
    for i in range(T):
        ref = IX.indexer_scores_row(q[i], w[i], K[ks[i]:ks[i] + nv[i]])
        tol = 1e-5 * np.max(np.abs(ref))
        assert np.max(np.abs(got[i, :nv[i]] - ref)) <= tol
        # exact on the kernel's own scores
        ref_idx, _ = IX.topk_row(got[i, :nv[i]].astype(np.float64), k)
        assert np.array_equal(gidx[i], ref_idx)
        # against the fp64 scores: everything clearly above the k-th score is selected,
        # and nothing selected is clearly below it
        kth = np.sort(ref)[::-1][k - 1]
        sel = set(gidx[i].tolist())
        assert all(j in sel for j in np.nonzero(ref > kth + 2 * tol)[0])
        assert all(ref[j] >= kth - 2 * tol for j in sel)
