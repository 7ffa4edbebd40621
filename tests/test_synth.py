"""The seeded input generator: its bf16 rounding and its determinism.

The generator feeds both the oracle and the CUDA path, so a change in it changes no parity
result; these tests keep its documented behaviour fixed."""

import numpy as np
import torch

from kv_token_compressor_b200 import synth


def test_round_to_bf16_matches_torch_conversion():
    # torch's fp32 -> bf16 conversion rounds to nearest, ties to even: an independent
    # implementation of the same rounding.  Random bit patterns cover every exponent,
    # subnormals, infinities and NaNs; the special values and ties are added by hand.
    rng = np.random.default_rng(7)
    u = rng.integers(0, 1 << 32, size=1 << 20, dtype=np.uint64).astype(np.uint32)
    special = np.array([0x00000000, 0x80000000, 0x00000001, 0x00008000, 0x00018000,
                        0x3F808000, 0x3F818000, 0x3F80FFFF, 0x7F7FFFFF, 0x7F7F8000,
                        0x7F7F7FFF, 0xFF7FFFFF, 0x7F800000, 0xFF800000, 0x7FC00000,
                        0x7F800001, 0xFFFFFFFF, 0xFFFF8000], dtype=np.uint32)
    u = np.concatenate([u, special])
    x = u.view(np.float32)
    got = synth.round_to_bf16(x)
    ref = torch.from_numpy(x.copy()).to(torch.bfloat16).to(torch.float32).numpy()
    nan = np.isnan(x)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))
    assert np.all(got.view(np.uint32) & 0xFFFF == 0)
    assert np.array_equal(x.view(np.uint32), u)  # the input is left as it was


def test_stream_inputs_are_seeded_and_bf16_valued():
    a = synth.stream_inputs("csa", 2, 64, 32, 4, "bf16", seed=3, z_row_offset=4.0)
    b = synth.stream_inputs("csa", 2, 64, 32, 4, "bf16", seed=3, z_row_offset=4.0)
    c = synth.stream_inputs("csa", 2, 64, 32, 4, "bf16", seed=4, z_row_offset=4.0)
    for k in ("Ca", "Cb", "Za", "Zb", "Ba", "Bb"):
        assert a[k].dtype == np.float32 and np.array_equal(a[k], b[k]), k
        assert not np.array_equal(a[k], c[k]), k
    for k in ("Ca", "Cb", "Za", "Zb"):
        assert a[k].shape == (2, 64, 32)
        assert np.all(a[k].view(np.uint32) & 0xFFFF == 0), k  # bf16 values
    assert a["Ba"].shape == (4, 32)


def test_torch_generators_shapes_dtypes_and_seeding():
    # The device-side generators (used by the full-size GPU tests and the bench) run on any
    # torch device; on the CPU their shapes, dtypes, seeding and ranges are checked here.
    dev = "cpu"
    a = synth.stream_inputs_torch("csa", 2, 256, 64, 4, "bf16", seed=1, z_row_offset=4.0, device=dev)
    b = synth.stream_inputs_torch("csa", 2, 256, 64, 4, "bf16", seed=1, z_row_offset=4.0, device=dev)
    for k in ("Ca", "Cb", "Za", "Zb"):
        assert a[k].shape == (2, 256, 64) and a[k].dtype == torch.bfloat16
        assert torch.equal(a[k], b[k])
    for k in ("Ba", "Bb"):
        assert a[k].shape == (4, 64) and a[k].dtype == torch.float32
    # the logit rows carry one offset U(-4, 4) each: row means spread far wider than C's
    za_means = a["Za"].float().mean(-1)
    assert za_means.abs().max() > 2.0 and a["Ca"].float().mean(-1).abs().max() < 1.0
    assert abs(a["Ba"].std().item() - 0.1 ** 0.5) < 0.05
    h = synth.stream_inputs_torch("hca", 1, 512, 32, 128, "f32", seed=2, device=dev)
    assert set(h) == {"C", "Z", "B"} and h["C"].dtype == torch.float32 and h["B"].shape == (128, 32)

    f = synth.fused_inputs_torch("csa", 1, 64, 256, 128, 4, seed=3, device=dev)
    assert f["H"].shape == (64, 256) and f["H"].dtype == torch.bfloat16
    for k in ("W_kva", "W_kvb", "W_za", "W_zb"):
        assert f[k].shape == (256, 128) and f[k].dtype == torch.bfloat16
    # W ~ N(0, 1/d): unit-variance projections
    assert abs(f["W_kva"].float().std().item() * 256 ** 0.5 - 1.0) < 0.05
    fh = synth.fused_inputs_torch("hca", 2, 128, 128, 128, 128, seed=3, device=dev)
    assert fh["H"].shape == (256, 128) and set(fh) == {"H", "W_kv", "W_z", "B"}

    s = synth.scalar_inputs_torch("csa", 1, 64, 32, 4, "bf16", seed=4, device=dev)
    assert s["za"].shape == (1, 64) and s["za"].dtype == torch.bfloat16 and s["ba"].shape == (4,)

    ix = synth.indexer_inputs_torch(3, 8, 100, seed=5, device=dev)
    assert ix["q"].shape == (3, 8, 128) and ix["q"].dtype == torch.bfloat16
    assert ix["K"].shape == (100, 128) and ix["w"].shape == (3, 8) and ix["w"].dtype == torch.float32
