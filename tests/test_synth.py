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
